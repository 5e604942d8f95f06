// Backward ring-attention kernels for sm_100a.
//
// The pages ("精读笔记 · Ring Attention with Blockwise Transformers for Near-Infinite
// Context", §4.2 and the BPT background of §2.2) state that training runs through the same
// blockwise ring structure but give no formulas; this is the analytic softmax gradient with
// P recomputed from the forward's log-sum-exp:
//   P = exp(scale q k^T - lse), dV = P^T dO, dP = dO V^T, Delta = rowsum(dO * O),
//   dS = P * (dP - Delta), dQ = scale dS K, dK = scale dS^T Q.
//
// Three kernels:
//   bwd_pre     -Delta (fp32) and -lse * log2(e) (fp32), both padded per head to a multiple
//               of 128 rows, and a zeroed fp32 dQ accumulator (HBM-bound).  Stored negated
//               so the key-row warpgroup's elementwise work is one packed add/FMA per pair.
//   bwd_kernel  key/value-stationary: one CTA per (head, 128-key tile) at a time, visiting
//               the query tiles that can see the key tile in ring order (ring step t brings
//               the key/value block j to the position of query block (j + t) mod D, step 0
//               being its own block); dK, dV accumulate in TMEM, dQ partials are added to
//               the fp32 accumulator by TMA bulk reduce-add.
//   bwd_convert dQ = scale * accumulator -> bf16 (HBM-bound).
//
// bwd_kernel<HD> CTA (512 threads; head dimension HD = 64 or 128):
//   warpgroups 0, 1  thread = key row, warpgroup h taking query columns [64h, 64h + 64): P^T,
//                dS^T (bf16) into TMEM and dS into shared memory; final dK, dV epilogue (head
//                columns [HD/2 h, HD/2 (h + 1))).  Each writes TMEM only inside columns it has
//                itself read, so the two never race.
//   warpgroup 2  thread = query row: reads dQ from TMEM, stages it (fp32, HD/32 128-B swizzled
//                boxes of 32 columns x 128 rows) over the query tile's own Q/dO stage once dK
//                has read Q, and one thread issues the TMA reduce-adds into the fp32
//                accumulator and then hands the stage back to the producer.
//   warp 12      TMA producer: K, V once per item; Q, dO, lse2, Delta per query tile (2 stages).
//   warp 13      TMEM allocator + tcgen05.mma issuer (warps 14, 15 complete warpgroup 3).
// TMEM (512 columns): [0,128) S^T, then P^T (bf16) of queries 0-63 in [0,32) and of queries
//   64-127 in [96,128); [128,256) dP^T, then dS^T in [128,160) and [224,256), then dQ (HD
//   columns) once dK has consumed dS^T; [256, 256 + HD) dV; [256 + HD, 256 + 2 HD) dK.
// MMAs per query tile (M = 128; in this order): S^T = K Q^T (N = 128, K = HD), dP^T = V dO^T,
//   dV += P^T dO (N = HD, K = 128), dK += dS^T Q, dQ = dS K (N = HD, K = 128).  The tensor
//   pipe executes them in issue order, so a later MMA may overwrite TMEM an earlier one reads:
//   S^T of the next tile is issued right after dQ (P^T is dead once dV issued), and only its
//   dP^T waits for the dQ readout.
#pragma once
#include <type_traits>

#include "ra_schedule.h"
#include "ra_sm100.cuh"
#include "ra_work.cuh"

namespace ra {
namespace bwd {

constexpr int BM = 128;   // keys per CTA tile (TMEM lanes of S^T, dP^T, dV, dK)
constexpr int BQ = 128;   // queries per query tile
constexpr int NSTAGE = 2;
constexpr int NUM_THREADS = 512;
constexpr int WARP_TMA = 12, WARP_MMA = 13;
// Registers: launched at 65536 / 512 = 128.  Warpgroup 3 (TMA, MMA, idle) lowers to
// REGS_OTHER; the key-row warpgroups raise to REGS_KEYS and the dQ warpgroup (128 fp32 dQ
// values per thread) to REGS_DQ.  The raises must not exceed what warpgroup 3 returns.
// 136 / 152 / 80 is the split with no spill anywhere: below 80 the TMA/MMA code spills, and
// a local-memory load in the MMA issue path leaves the tensor pipe idle (3 % slower at 56).
#ifndef RA_BWD_REGS_KEYS
#define RA_BWD_REGS_KEYS 136
#define RA_BWD_REGS_DQ 152
#define RA_BWD_REGS_OTHER 80
#endif
constexpr uint32_t REGS_LAUNCH = 128;
constexpr uint32_t REGS_KEYS = RA_BWD_REGS_KEYS, REGS_DQ = RA_BWD_REGS_DQ, REGS_OTHER = RA_BWD_REGS_OTHER;
static_assert(2 * (REGS_KEYS - REGS_LAUNCH) + (REGS_DQ - REGS_LAUNCH) <= REGS_LAUNCH - REGS_OTHER,
              "register split exceeds the pool");
static_assert(NUM_THREADS * REGS_LAUNCH <= 65536, "launch register budget");
constexpr uint32_t TMEM_COLS = 512;
// Of every 8 columns of P, 2 x this many exponentials run on the FMA pipes (exp2_fma2).
// 0 by default: with four warpgroups the MUFU pipe keeps up, and moving exponentials to
// the FMA pipes measured 8% slower at S = 16K, Dh = 128.
#ifndef RA_BWD_EXP2_FMA_PER4
#define RA_BWD_EXP2_FMA_PER4 0
#endif
constexpr uint32_t COL_S = 0, COL_DP = 128, COL_DQ = 128, COL_DV = 256;
template <int HD>
__host__ __device__ constexpr uint32_t col_dk() { return COL_DV + HD; }
// bf16 P^T / dS^T of query columns [64h, 64h + 64): TMEM columns [base, base + 32)
__host__ __device__ constexpr uint32_t col_p(int h) { return h ? 96u : 0u; }
__host__ __device__ constexpr uint32_t col_ds(int h) { return h ? 224u : 128u; }

template <int HD>
struct Layout {
  static_assert(HD == 64 || HD == 128, "head dim");
  static constexpr int SUB = HD / 64;                  // 128-byte-swizzled column blocks of a tile
  static constexpr int SUB_BYTES = 128 * 128;          // 128 rows x 128 B (64 bf16)
  static constexpr int TILE_BYTES = SUB * SUB_BYTES;   // 128 rows x HD bf16
  static constexpr int DS_BYTES = 2 * SUB_BYTES;       // 128 keys x 128 queries bf16
  static constexpr int K_OFF = 0;
  static constexpr int V_OFF = K_OFF + TILE_BYTES;
  static constexpr int DS_OFF = V_OFF + TILE_BYTES;    // dS, MN-major: two 64-query halves
  static constexpr int STAGE_OFF = DS_OFF + DS_BYTES;
  static constexpr int STAGE_Q = 0, STAGE_DO = TILE_BYTES, STAGE_LSE = 2 * TILE_BYTES,
                       STAGE_DELTA = STAGE_LSE + BQ * 4, STAGE_BYTES = STAGE_DELTA + BQ * 4;
  static constexpr int BAR_OFF = STAGE_OFF + NSTAGE * STAGE_BYTES;
  static constexpr int B_KV_FULL = 0, B_KV_EMPTY = 1, B_QD_FULL = 2, B_QD_EMPTY = B_QD_FULL + NSTAGE,
                       B_S_FULL = B_QD_EMPTY + NSTAGE, B_DP_FULL = B_S_FULL + 1, B_P_READY = B_DP_FULL + 1,
                       B_DS_READY = B_P_READY + 1, B_DQ_FULL = B_DS_READY + 1, B_DQ_FREE = B_DQ_FULL + 1,
                       B_ACC_FULL = B_DQ_FREE + 1, B_DK_DONE = B_ACC_FULL + 1, B_DRAIN = B_DK_DONE + 1,
                       B_WQ_FULL = B_DRAIN + 1, B_WQ_EMPTY = B_WQ_FULL + 2, NUM_BARS = B_WQ_EMPTY + 2;
  static constexpr uint32_t WQ_CONSUMERS = 1 + 12;   // MMA thread + one arrival per warp of warpgroups 0-2
  static constexpr int MISC_OFF = BAR_OFF + NUM_BARS * 8;   // TMEM base, abort flag, item ring[2]
  static constexpr int BYTES = MISC_OFF + 16;
  // the dQ staging (HD/32 boxes of 128 rows x 128 B) fits over a stage's Q and dO tiles
  static_assert((HD / 32) * SUB_BYTES <= 2 * TILE_BYTES, "dQ staging");
  static_assert(STAGE_BYTES % 1024 == 0 && STAGE_OFF % 1024 == 0, "swizzled tiles need 1024-B alignment");
};
static_assert(Layout<128>::BYTES <= 232448 && Layout<64>::BYTES <= 232448, "shared memory");

struct Params {
  int BH, S, S_pad, D, causal;
  int n_kt;              // key tiles per head
  int n_items;           // BH * n_kt
  int hgroup;            // heads whose items are interleaved (L2 reuse of Q, dO)
  int work_slot;         // this launch's work counter
  float scale_log2;      // scale * log2(e)
  float scale;
  const float* lse2;     // [BH][S_pad] -lse * log2(e), -inf in padding
  const float* delta;    // [BH][S_pad] -Delta
  float* dq_acc;         // [BH][S][HD] fp32
  __nv_bfloat16* dk;     // [BH][S][HD]
  __nv_bfloat16* dv;
  float* dk32;           // non-null: dK, dV are added to these fp32 [BH][S][HD] instead of
  float* dv32;           // written to dk, dv (rows of a key tile belong to one CTA)
};

using RingQTiles = ::ra::RingQTiles;

// Work item w -> (bh, key tile).  Heads are taken in groups of p.hgroup whose Q/dO fit in
// L2 together; inside a group items go key tile by key tile (causal: the first key tiles
// see the most query tiles, so the longest items come first).
__device__ __forceinline__ void item_coords(int w, const Params& p, int& bh, int& kt) {
  const int per_group = p.hgroup * p.n_kt;
  const int g = w / per_group;
  const int gsize = min(p.hgroup, p.BH - g * p.hgroup);
  const int idx = w - g * per_group;
  kt = idx / gsize;
  bh = g * p.hgroup + (idx - kt * gsize);
}

__device__ __forceinline__ void advance(int& stage, uint32_t& phase) {
  if (++stage == NSTAGE) {
    stage = 0;
    phase ^= 1u;
  }
}

// ------------------------------------------------------------------ producer
template <int HD>
__device__ void producer(const CUtensorMap* tm_q, const CUtensorMap* tm_k, const CUtensorMap* tm_v,
                         const CUtensorMap* tm_do, const Params& p, uint32_t sbase, volatile int* wq,
                         volatile int* abort_flag) {
  using L = Layout<HD>;
  auto bar = [&](int i) { return sbase + L::BAR_OFF + 8u * i; };
  int stage = 0;
  uint32_t phase = 0, kv_phase = 0;
  uint32_t issued = 0, issued_parity = 0, kv_issued = 0, kv_parity = 0;
  bool ok = true;
  ItemRing ring{bar(L::B_WQ_FULL), bar(L::B_WQ_EMPTY), wq};
  int w = work_fetch(p.work_slot);
  for (;;) {
    if (!ring.push(w, abort_flag)) { ok = false; break; }
    if (w >= p.n_items) break;
    const int w_next = work_fetch(p.work_slot);
    int bh, kt;
    item_coords(w, p, bh, kt);
    if (!mbar_wait(bar(L::B_KV_EMPTY), kv_phase ^ 1u, abort_flag)) { ok = false; break; }
    mbar_arrive_expect_tx(bar(L::B_KV_FULL), 2 * L::TILE_BYTES);
    for (int sb = 0; sb < L::SUB; ++sb) {
      tma_load_3d(tm_k, sbase + L::K_OFF + sb * L::SUB_BYTES, bar(L::B_KV_FULL), sb * 64, kt * BM, bh);
      tma_load_3d(tm_v, sbase + L::V_OFF + sb * L::SUB_BYTES, bar(L::B_KV_FULL), sb * 64, kt * BM, bh);
    }
    kv_issued = 1;
    kv_parity = kv_phase;
    kv_phase ^= 1u;
    RingQTiles it;
    it.init(p.S, p.D, p.causal, kt * BM, BQ);
    for (int qt = it.next(); qt >= 0; qt = it.next()) {
      if (!mbar_wait(bar(L::B_QD_EMPTY + stage), phase ^ 1u, abort_flag)) { ok = false; break; }
      const uint32_t full = bar(L::B_QD_FULL + stage);
      const uint32_t st = sbase + L::STAGE_OFF + stage * L::STAGE_BYTES;
      mbar_arrive_expect_tx(full, 2 * L::TILE_BYTES + 2 * BQ * 4);
      for (int sb = 0; sb < L::SUB; ++sb) {
        tma_load_3d(tm_q, st + L::STAGE_Q + sb * L::SUB_BYTES, full, sb * 64, qt * BQ, bh);
        tma_load_3d(tm_do, st + L::STAGE_DO + sb * L::SUB_BYTES, full, sb * 64, qt * BQ, bh);
      }
      const size_t row0 = static_cast<size_t>(bh) * p.S_pad + static_cast<size_t>(qt) * BQ;
      bulk_load(st + L::STAGE_LSE, p.lse2 + row0, BQ * 4, full);
      bulk_load(st + L::STAGE_DELTA, p.delta + row0, BQ * 4, full);
      issued |= 1u << stage;
      issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
      advance(stage, phase);
    }
    if (!ok) break;
    w = w_next;
  }
  work_done(p.work_slot);
  if (!ok) {
    for (int s = 0; s < NSTAGE; ++s)
      if (issued & (1u << s)) drain_wait(bar(L::B_QD_FULL + s), (issued_parity >> s) & 1u);
    if (kv_issued) drain_wait(bar(L::B_KV_FULL), kv_parity);
  }
}

// ------------------------------------------------------------------ MMA issuer
template <int HD>
__device__ __forceinline__ void mma_kmajor(uint32_t d_tmem, uint32_t a_smem, uint32_t b_smem, bool first_zero) {
  // D[128 x 128] = A[128 x HD] * B[128 x HD]^T, both K-major 128-B swizzled (64-column blocks)
  constexpr uint32_t IDESC = idesc_bf16_f32(128, 128, 0, 0);
#pragma unroll
  for (int kk = 0; kk < HD / 16; ++kk) {
    const uint32_t off = (kk >> 2) * Layout<HD>::SUB_BYTES + (kk & 3) * 32;
    umma_ss(d_tmem, sdesc_sw128(a_smem + off, 16, 1024), sdesc_sw128(b_smem + off, 16, 1024), IDESC,
            (first_zero && kk == 0) ? 0u : 1u);
  }
}

template <int HD>
__device__ __forceinline__ void mma_tmem_a(uint32_t d_tmem, uint32_t a_lo, uint32_t a_hi, uint32_t b_smem,
                                           bool accumulate) {
  // D[128 x HD] (+)= A[128 x 128] (TMEM, bf16; K = 0-63 at a_lo, 64-127 at a_hi)
  //                  * B[128 x HD] (smem, MN-major: rows = K, 64-column blocks SUB_BYTES apart)
  constexpr uint32_t IDESC = idesc_bf16_f32(128, HD, 0, 1);
#pragma unroll
  for (int kk = 0; kk < BQ / 16; ++kk)
    umma_ts(d_tmem, (kk < 4 ? a_lo : a_hi) + (kk & 3) * 8,
            sdesc_sw128(b_smem + kk * 2048, Layout<HD>::SUB_BYTES, 1024), IDESC, (accumulate || kk > 0) ? 1u : 0u);
}

template <int HD>
__device__ __forceinline__ void mma_dq(uint32_t d_tmem, uint32_t ds_smem, uint32_t k_smem) {
  // dQ [128 q x HD] = dS [128 q x 128 k] (MN-major: q contiguous, two 64-q halves)
  //                  * K [128 k x HD] (MN-major: rows = K, 64-column blocks)
  constexpr uint32_t IDESC = idesc_bf16_f32(128, HD, 1, 1);
#pragma unroll
  for (int kk = 0; kk < BM / 16; ++kk)
    umma_ss(d_tmem, sdesc_sw128(ds_smem + kk * 2048, Layout<HD>::SUB_BYTES, 1024),
            sdesc_sw128(k_smem + kk * 2048, Layout<HD>::SUB_BYTES, 1024), IDESC, kk > 0 ? 1u : 0u);
}

template <int HD>
__device__ void mma_issuer(const Params& p, uint32_t sbase, uint32_t tmem, volatile int* wq, volatile int* abort_flag) {
  using L = Layout<HD>;
  auto bar = [&](int i) { return sbase + L::BAR_OFF + 8u * i; };
  int stage = 0;
  uint32_t phase = 0, kv_phase = 0, p_phase = 0, ds_phase = 0, dqf_phase = 0;
  bool ok = true;
  bool dq_pending = false;   // a dQ readout of the previous query tile is outstanding
  ItemRing ring{bar(L::B_WQ_FULL), bar(L::B_WQ_EMPTY), wq};
  for (;;) {
    int w;
    if (!ring.pop(w, abort_flag)) { ok = false; break; }
    if (w >= p.n_items) break;
    int bh, kt;
    item_coords(w, p, bh, kt);
    if (!mbar_wait(bar(L::B_KV_FULL), kv_phase, abort_flag)) { ok = false; break; }
    kv_phase ^= 1u;
    tc_fence_after();
    RingQTiles it;
    it.init(p.S, p.D, p.causal, kt * BM, BQ);
    int n = 0;
    for (int qt = it.next(); qt >= 0; qt = it.next(), ++n) {
      const int s = stage;
      const uint32_t st = sbase + L::STAGE_OFF + s * L::STAGE_BYTES;
      if (!mbar_wait(bar(L::B_QD_FULL + s), phase, abort_flag)) { ok = false; break; }
      advance(stage, phase);
      tc_fence_after();
      mma_kmajor<HD>(tmem + COL_S, sbase + L::K_OFF, st + L::STAGE_Q, true);     // S^T = K Q^T
      tc_commit(bar(L::B_S_FULL));
      if (dq_pending) {  // dP^T overwrites the columns the previous tile's dQ readout reads
        if (!mbar_wait(bar(L::B_DQ_FREE), dqf_phase, abort_flag)) { ok = false; break; }
        dqf_phase ^= 1u;
        tc_fence_after();
      }
      mma_kmajor<HD>(tmem + COL_DP, sbase + L::V_OFF, st + L::STAGE_DO, true);   // dP^T = V dO^T
      tc_commit(bar(L::B_DP_FULL));
      if (!mbar_wait(bar(L::B_P_READY), p_phase, abort_flag)) { ok = false; break; }
      p_phase ^= 1u;
      tc_fence_after();
      mma_tmem_a<HD>(tmem + COL_DV, tmem + col_p(0), tmem + col_p(1), st + L::STAGE_DO, n > 0);   // dV += P^T dO
      if (!mbar_wait(bar(L::B_DS_READY), ds_phase, abort_flag)) { ok = false; break; }
      ds_phase ^= 1u;
      tc_fence_after();
      mma_tmem_a<HD>(tmem + col_dk<HD>(), tmem + col_ds(0), tmem + col_ds(1), st + L::STAGE_Q, n > 0);   // dK += dS^T Q
      tc_commit(bar(L::B_DK_DONE));   // Q and dO of this stage no longer read by the tensor core
      mma_dq<HD>(tmem + COL_DQ, sbase + L::DS_OFF, sbase + L::K_OFF);                 // dQ = dS K
      tc_commit(bar(L::B_DQ_FULL));
      dq_pending = true;
    }
    if (!ok) break;
    tc_commit(bar(L::B_ACC_FULL));   // dV, dK final once everything issued so far completes
    tc_commit(bar(L::B_KV_EMPTY));   // K, V (read by the last dQ MMAs) free then too
  }
  tc_commit(bar(L::B_DRAIN));
  drain_wait(bar(L::B_DRAIN), 0);
}

// ------------------------------------------------------------------ warpgroups 0, 1: P^T, dS^T, epilogue
template <int HD, int half>
__device__ void key_rows_wg(const Params& p, uint8_t* smem, uint32_t sbase, uint32_t tmem, volatile int* wq,
                            volatile int* abort_flag) {
  using L = Layout<HD>;
  auto bar = [&](int i) { return sbase + L::BAR_OFF + 8u * i; };
  const int lane = threadIdx.x & 31;
  const int quarter = (threadIdx.x >> 5) & 3;
  const int row = quarter * 32 + lane;   // key row within the tile
  constexpr int qc0 = 64 * half;         // this warpgroup's first query column
  const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
  const float2 sl2x2 = make_float2(p.scale_log2, p.scale_log2);
  int stage = 0;
  uint32_t phase = 0, s_phase = 0, dp_phase = 0, acc_phase = 0;
  // this thread's dS row in the MN-major shared tile: queries [qc0, qc0 + 64) form half
  // `half`; 16-B chunk j of the 128-B row is stored at chunk j ^ (row & 7) (128-B swizzle)
  uint8_t* ds_row = smem + L::DS_OFF + half * L::SUB_BYTES + row * 128;
  const int sw = row & 7;

  ItemRing ring{bar(L::B_WQ_FULL), bar(L::B_WQ_EMPTY), wq};
  for (;;) {
    int w = 0;
    if (!ring.pop_warp(w, abort_flag)) return;
    if (w >= p.n_items) break;
    int bh, kt;
    item_coords(w, p, bh, kt);
    const int k_row = kt * BM + row;
    RingQTiles it;
    it.init(p.S, p.D, p.causal, kt * BM, BQ);
    for (int qt = it.next(); qt >= 0; qt = it.next()) {
      const uint8_t* stg = smem + L::STAGE_OFF + stage * L::STAGE_BYTES;
      const float* nlse2 = reinterpret_cast<const float*>(stg + L::STAGE_LSE) + qc0;   // -lse * log2(e)
      const float* ndlt = reinterpret_cast<const float*>(stg + L::STAGE_DELTA) + qc0;  // -Delta
      const int q0 = qt * BQ + qc0;
      // visible queries of this key row: columns [lo, hi) of this warpgroup's 64
      const int lo = p.causal ? k_row - q0 : 0;
      const int hi = (k_row < p.S) ? p.S - q0 : 0;
      const bool masked = (lo > 0) || (hi < 64);

      // ---- P^T = exp2(S^T * scale * log2e - lse * log2e)
      // lse2 / Delta arrive by bulk copy on the stage's full barrier: observe it directly
      bool ok = mbar_wait(bar(L::B_QD_FULL + stage), phase, abort_flag);
      ok = ok && mbar_wait(bar(L::B_S_FULL), s_phase, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) return;
      advance(stage, phase);
      s_phase ^= 1u;
      tc_fence_after();
      float pv[64];
      {
        uint32_t r[64];
        tmem_ld32(lane_base + COL_S + qc0, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
        tmem_ld32(lane_base + COL_S + qc0 + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < 64; c += 4) {
          const float4 l4 = *reinterpret_cast<const float4*>(nlse2 + c);
          const float2 xa = __ffma2_rn(make_float2(__uint_as_float(r[c]), __uint_as_float(r[c + 1])), sl2x2,
                                       make_float2(l4.x, l4.y));
          const float2 xb = __ffma2_rn(make_float2(__uint_as_float(r[c + 2]), __uint_as_float(r[c + 3])), sl2x2,
                                       make_float2(l4.z, l4.w));
          float2 pa, pb;
          if (((c >> 2) & 1) < RA_BWD_EXP2_FMA_PER4) {
            pa = exp2_fma2(xa);
          } else {
            pa.x = ex2_approx(xa.x);
            pa.y = ex2_approx(xa.y);
          }
          pb.x = ex2_approx(xb.x);
          pb.y = ex2_approx(xb.y);
          pv[c] = pa.x;
          pv[c + 1] = pa.y;
          pv[c + 2] = pb.x;
          pv[c + 3] = pb.y;
        }
      }
      if (masked) {
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (c < lo || c >= hi) pv[c] = 0.f;
      }
      {
        uint32_t pk[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) pk[c] = pack_bf16x2(pv[2 * c], pv[2 * c + 1]);
        tmem_st32(lane_base + col_p(half), pk);   // inside the S^T columns this warpgroup read
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(L::B_P_READY));

      // ---- dS^T = P^T * (dP^T - Delta), 32 query columns at a time.  dS^T goes to columns
      // this warpgroup has already read: warpgroup 1 walks its chunks from the high end.
      // (the previous tile's dQ MMA, the last reader of the dS buffer, completed before the dQ
      // readout released the TMEM columns that this tile's dP^T was then written into)
      ok = mbar_wait(bar(L::B_DP_FULL), dp_phase, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) return;
      dp_phase ^= 1u;
      tc_fence_after();
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int ch = half ? 1 - i : i;   // chunk = query columns [32 ch, 32 ch + 32) of this half (compile time)
        uint32_t d[32];
        tmem_ld32(lane_base + COL_DP + qc0 + 32 * ch, d);
        tmem_ld_wait();
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          const float2 nd = *reinterpret_cast<const float2*>(ndlt + 32 * ch + c);
          const float2 g = __fmul2_rn(make_float2(pv[32 * ch + c], pv[32 * ch + c + 1]),
                                      __fadd2_rn(make_float2(__uint_as_float(d[c]), __uint_as_float(d[c + 1])), nd));
          pk[c >> 1] = pack_bf16x2(g.x, g.y);
        }
        tmem_st16(lane_base + col_ds(half) + 16 * ch, pk);
#pragma unroll
        for (int j = 0; j < 4; ++j)
          *reinterpret_cast<uint4*>(ds_row + (((4 * ch + j) ^ sw) << 4)) =
              make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
      }
      tmem_st_wait();
      fence_proxy_async_smem();   // generic-proxy dS stores -> visible to the tensor core
      tc_fence_before();
      mbar_arrive(bar(L::B_DS_READY));
    }
    // ---- epilogue: dV, dK (scaled), head columns [HD/2 half, HD/2 (half + 1))
    if (!__all_sync(0xffffffffu, mbar_wait(bar(L::B_ACC_FULL), acc_phase, abort_flag))) return;
    acc_phase ^= 1u;
    tc_fence_after();
    constexpr int hc0 = (HD / 2) * half;   // this warpgroup's first head column
    const bool row_ok = k_row < p.S;
    const size_t off = (static_cast<size_t>(bh) * p.S + k_row) * HD + hc0;
#pragma unroll
    for (int which = 0; which < 2; ++which) {
      const uint32_t col = (which ? col_dk<HD>() : COL_DV) + hc0;
      const float mul = which ? p.scale : 1.f;
      __nv_bfloat16* dst_row = (which ? p.dk : p.dv) + off;
#pragma unroll
      for (int c = 0; c < HD / 64; ++c) {
        uint32_t rr[32];
        tmem_ld32(lane_base + col + 32 * c, rr);
        tmem_ld_wait();
        if (p.dk32 != nullptr) {   // uniform: accumulate in fp32
          if (row_ok) {
            float4* acc = reinterpret_cast<float4*>((which ? p.dk32 : p.dv32) + off + 32 * c);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              float4 a = acc[i];
              a.x = fmaf(__uint_as_float(rr[4 * i]), mul, a.x);
              a.y = fmaf(__uint_as_float(rr[4 * i + 1]), mul, a.y);
              a.z = fmaf(__uint_as_float(rr[4 * i + 2]), mul, a.z);
              a.w = fmaf(__uint_as_float(rr[4 * i + 3]), mul, a.w);
              acc[i] = a;
            }
          }
          continue;
        }
        uint32_t w16[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          w16[i] = pack_bf16x2(__uint_as_float(rr[2 * i]) * mul, __uint_as_float(rr[2 * i + 1]) * mul);
        if (row_ok) {
          uint4* dst = reinterpret_cast<uint4*>(dst_row + 32 * c);
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w16[4 * i], w16[4 * i + 1], w16[4 * i + 2], w16[4 * i + 3]);
        }
      }
    }
  }
}

// ------------------------------------------------------------------ warpgroup 2: dQ readout
template <int HD>
__device__ void query_rows_wg(const Params& p, const CUtensorMap* tm_dq, uint8_t* smem, uint32_t sbase, uint32_t tmem,
                              volatile int* wq, volatile int* abort_flag) {
  using L = Layout<HD>;
  auto bar = [&](int i) { return sbase + L::BAR_OFF + 8u * i; };
  const int lane = threadIdx.x & 31;
  const int quarter = (threadIdx.x >> 5) & 3;
  const int row = quarter * 32 + lane;   // query row within the tile
  const bool leader = (threadIdx.x & 127) == 0;
  const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
  const int sw = row & 7;
  uint32_t phase = 0, dk_phase = 0, qphase = 0;
  int stage = 0;
  bool ok = true;
  ItemRing ring{bar(L::B_WQ_FULL), bar(L::B_WQ_EMPTY), wq};
  for (;;) {
    int w = 0;
    // warpgroup-uniform outcome (the named barriers below need all four warps)
    ok = named_bar_and(1, 128, ring.pop_warp(w, abort_flag));
    if (!ok || w >= p.n_items) break;
    int bh, kt;
    item_coords(w, p, bh, kt);
    RingQTiles it;
    it.init(p.S, p.D, p.causal, kt * BM, BQ);
    for (int qt = it.next(); qt >= 0; qt = it.next()) {
      // every thread of the warpgroup reaches this barrier (the wait is bounded), so the
      // named barriers below never wait for a thread that gave up
      ok = named_bar_and(1, 128, mbar_wait(bar(L::B_DQ_FULL), phase, abort_flag));
      if (!ok) break;
      phase ^= 1u;
      tc_fence_after();
      uint32_t r[HD];
#pragma unroll
      for (int c = 0; c < HD / 32; ++c) tmem_ld32(lane_base + COL_DQ + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&r[32 * c]));
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(bar(L::B_DQ_FREE));   // dQ is in registers: hand the TMEM columns back
      // the tile's Q/dO stage becomes staging once dK (the last MMA reading Q) has completed
      ok = named_bar_and(1, 128, mbar_wait(bar(L::B_DK_DONE), dk_phase, abort_flag));
      if (!ok) break;
      dk_phase ^= 1u;
      const int s_idx = stage;
      if (++stage == NSTAGE) {
        stage = 0;
        qphase ^= 1u;
      }
      // dQ row -> HD/32 32-column fp32 boxes (128 B per row, 128-B swizzle) over Q and dO
      uint8_t* st_row = smem + L::STAGE_OFF + s_idx * L::STAGE_BYTES + row * 128;
#pragma unroll
      for (int b = 0; b < HD / 32; ++b)
#pragma unroll
        for (int j = 0; j < 8; ++j)
          *reinterpret_cast<uint4*>(st_row + b * L::SUB_BYTES + ((j ^ sw) << 4)) =
              make_uint4(r[32 * b + 4 * j], r[32 * b + 4 * j + 1], r[32 * b + 4 * j + 2], r[32 * b + 4 * j + 3]);
      fence_proxy_async_smem();
      named_bar_sync(1, 128);
      if (leader) {
        const uint32_t st = sbase + L::STAGE_OFF + s_idx * L::STAGE_BYTES;
#pragma unroll
        for (int b = 0; b < HD / 32; ++b) tma_reduce_add_3d(tm_dq, st + b * L::SUB_BYTES, 32 * b, qt * BQ, bh);
        bulk_commit();
        bulk_wait_read_all();
        mbar_arrive(bar(L::B_QD_EMPTY + s_idx));   // the producer may refill this stage
      }
    }
    if (!ok) break;
  }
  if (leader) bulk_wait_all();   // reduce-adds complete before the CTA exits
}

// ------------------------------------------------------------------ main kernel
template <int HD>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
               const __grid_constant__ CUtensorMap tm_dq, const Params p) {
  using L = Layout<HD>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 4);
  volatile int* wq = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 8);
  const int warp = threadIdx.x >> 5;
  if (sbase & 1023u) {   // the 128-byte swizzle needs 1024-byte aligned tiles
    if (threadIdx.x == 0) record_status(RA_ERR_CUDA);
    return;              // uniform: every thread sees the same base
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < L::NUM_BARS; ++i) {
      const bool key_rows = (i == L::B_P_READY || i == L::B_DS_READY);   // both key-row warpgroups
      const bool wq_empty = (i >= L::B_WQ_EMPTY && i < L::B_WQ_EMPTY + 2);
      const uint32_t count = key_rows ? 256 : (i == L::B_DQ_FREE ? 128 : (wq_empty ? L::WQ_CONSUMERS : 1));
      mbar_init(sbase + L::BAR_OFF + 8u * i, count);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == WARP_MMA) {
    tmem_alloc(smem_u32(tmem_holder), TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == WARP_TMA && (threadIdx.x & 31) == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_do);
    tma_prefetch_desc(&tm_dq);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp >= 12) {
    regs_lower<REGS_OTHER>();
    if (warp == WARP_TMA) {
      if ((threadIdx.x & 31) == 0) producer<HD>(&tm_q, &tm_k, &tm_v, &tm_do, p, sbase, wq, abort_flag);
      __syncwarp();
    } else if (warp == WARP_MMA) {
      if ((threadIdx.x & 31) == 0) mma_issuer<HD>(p, sbase, tmem, wq, abort_flag);
      __syncwarp();
    }
  } else if (warp < 8) {
    regs_raise<REGS_KEYS>();
    if (warp < 4)
      key_rows_wg<HD, 0>(p, smem, sbase, tmem, wq, abort_flag);
    else
      key_rows_wg<HD, 1>(p, smem, sbase, tmem, wq, abort_flag);
  } else {
    regs_raise<REGS_DQ>();
    query_rows_wg<HD>(p, &tm_dq, smem, sbase, tmem, wq, abort_flag);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == WARP_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// ------------------------------------------------------------------ preprocess / convert
constexpr int PRE_WARPS = 8;

// One warp per padded row: -Delta = -sum_d dO * O and -lse * log2(e) (0 and -inf in the
// padding rows), and the row of the fp32 dQ accumulator cleared.  HD / 32 values per lane.
template <int HD>
__global__ void __launch_bounds__(PRE_WARPS * 32)
    bwd_pre_kernel(const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ dO,
                   const float* __restrict__ lse, float* __restrict__ delta, float* __restrict__ lse2,
                   float* __restrict__ dq_acc, int BH, int S, int S_pad) {
  const int lane = threadIdx.x & 31;
  const long long prow = static_cast<long long>(blockIdx.x) * PRE_WARPS + (threadIdx.x >> 5);
  if (prow >= static_cast<long long>(BH) * S_pad) return;
  const long long bh = prow / S_pad;
  const int s = static_cast<int>(prow - bh * S_pad);
  if (s >= S) {
    if (lane == 0) {
      delta[prow] = 0.f;
      lse2[prow] = -INFINITY;
    }
    return;
  }
  const long long row = bh * S + s;
  constexpr int PER_LANE = HD / 32;   // bf16 values of a row per lane: 4 (8 bytes) or 2 (4 bytes)
  using Vec = typename std::conditional<PER_LANE == 4, uint2, uint32_t>::type;
  const Vec a = __ldg(reinterpret_cast<const Vec*>(o + row * HD) + lane);
  const Vec b = __ldg(reinterpret_cast<const Vec*>(dO + row * HD) + lane);
  const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
  const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&b);
  float acc = 0.f;
#pragma unroll
  for (int i = 0; i < PER_LANE / 2; ++i) {
    const float2 fa = __bfloat1622float2(a2[i]), fb = __bfloat1622float2(b2[i]);
    acc = fmaf(fa.x, fb.x, acc);
    acc = fmaf(fa.y, fb.y, acc);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if constexpr (PER_LANE == 4)
    reinterpret_cast<float4*>(dq_acc + row * HD)[lane] = make_float4(0.f, 0.f, 0.f, 0.f);
  else
    reinterpret_cast<float2*>(dq_acc + row * HD)[lane] = make_float2(0.f, 0.f);
  if (lane == 0) {
    delta[prow] = -acc;
    lse2[prow] = -lse[row] * 1.4426950408889634f;
  }
}

// dQ = scale * accumulator -> bf16, 8 elements per thread.
__global__ void __launch_bounds__(256)
    bwd_convert_kernel(const float* __restrict__ dq_acc, __nv_bfloat16* __restrict__ dq, long long n8, float scale) {
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n8) return;
  const float4 a = __ldg(reinterpret_cast<const float4*>(dq_acc) + 2 * i);
  const float4 b = __ldg(reinterpret_cast<const float4*>(dq_acc) + 2 * i + 1);
  reinterpret_cast<uint4*>(dq)[i] = make_uint4(pack_bf16x2(a.x * scale, a.y * scale), pack_bf16x2(a.z * scale, a.w * scale),
                                               pack_bf16x2(b.x * scale, b.y * scale), pack_bf16x2(b.z * scale, b.w * scale));
}

// dQ32 += scale * accumulator (fp32), 4 elements per thread.
__global__ void __launch_bounds__(256)
    bwd_accum_dq_kernel(const float* __restrict__ dq_acc, float* __restrict__ dq32, long long n4, float scale) {
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n4) return;
  const float4 a = __ldg(reinterpret_cast<const float4*>(dq_acc) + i);
  float4 d = reinterpret_cast<const float4*>(dq32)[i];
  d.x = fmaf(a.x, scale, d.x);
  d.y = fmaf(a.y, scale, d.y);
  d.z = fmaf(a.z, scale, d.z);
  d.w = fmaf(a.w, scale, d.w);
  reinterpret_cast<float4*>(dq32)[i] = d;
}

}  // namespace bwd
}  // namespace ra
