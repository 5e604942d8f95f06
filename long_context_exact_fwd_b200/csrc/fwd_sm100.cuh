// Forward ring-attention kernel for sm_100a: TMA-staged K/V ring buffer, tcgen05 MMAs with
// TMEM accumulators, one thread per query row for the online softmax.
//
// Pages: "精读笔记 · Ring Attention with Blockwise Transformers for Near-Infinite Context"
// §3.1 (a query block against key/value blocks in any order, statistics combined with
// rescaling), §3.2/§3.5 (ring order, step 0 = own block), §3.3 (block transfer overlapped
// with block compute -- here the on-chip analogue: the K/V tiles of the next steps are in
// flight through TMA while the tensor cores work on the current one).
//
// CTA = one work item at a time (persistent grid; items taken from a global counter):
//   item = (b*H + h, pair of query tiles Q0 = rows [256i, 256i+128), Q1 = the next 128).
//   warps 0-3  softmax for Q0 (thread = row = TMEM lane), warps 4-7 softmax for Q1,
//   warp 8     TMA producer (Q pair, then K_j, V_j per key tile into an NSTAGE ring),
//   warp 9     TMEM allocator + single-thread tcgen05.mma issuer.
// TMEM (512 columns): S0 | S1 | O0 | O1, 128 fp32 columns each; P_t (bf16) overwrites the
// first 64 columns of S_t and feeds O_t += P_t V as the A operand straight from TMEM.
// Issue order per key tile j (ping-pong, so the softmax of one query tile overlaps the
// tensor-core work of the other):
//   O0 += P0(j-1) V(j-1);  S0 = Q0 K(j)^T;  O1 += P1(j-1) V(j-1);  S1 = Q1 K(j)^T.
// SPLIT = true (ring_attn_fwd_split): a work item is one piece of a pair's visit order
// (RingTiles::restrict_to); the epilogue writes the piece's normalised fp32 O and its lse
// for the merge instead of bf16 O.
// Online softmax (base 2, scale folded in): the running max used as exponent reference is
// only raised when the tile max exceeds it by more than 8 (a factor 256), so O is rescaled
// in TMEM rarely; any reference gives the same O / l exactly in real arithmetic.
#pragma once
#include "ra_schedule.h"
#include "ra_sm100.cuh"
#include "ra_work.cuh"

namespace ra {
namespace fwd {

constexpr int BM = 128;        // query rows per tile (= TMEM lanes)
constexpr int BN = 128;        // keys per key/value tile
constexpr int NQ = 2;          // query tiles per CTA
constexpr int ROWS = BM * NQ;  // query rows per work item
constexpr int NSTAGE = 4;      // K/V shared-memory stages (each holds one K or one V tile)
constexpr int NUM_THREADS = 384;   // three full warpgroups (registers are granted per warpgroup)
constexpr int WARP_TMA = 8;
constexpr int WARP_MMA = 9;        // warps 10-11 only complete the third warpgroup
// Register split: launched at 65536 / 384 = 168 per thread.  Warpgroup 2 (TMA, MMA) lowers
// to 104, freeing 128 x 64; the two softmax warpgroups raise to 200, taking 2 x 128 x 32 =
// 128 x 64.  The raises exactly equal the lowers.  At 88 the TMA/MMA code spilled to local
// memory (a load in the MMA issue path stalls the tensor pipe); 200 is enough for softmax.
constexpr uint32_t REGS_LAUNCH = 168, REGS_SOFTMAX = 200, REGS_OTHER = 104;
static_assert(2 * (REGS_SOFTMAX - REGS_LAUNCH) <= REGS_LAUNCH - REGS_OTHER, "register split exceeds the pool");
static_assert(NUM_THREADS * REGS_LAUNCH <= 65536, "launch register budget");
constexpr float RESCALE_LOG2 = 8.0f;
// Of every 4 exponential pairs of a row, this many are evaluated on the FMA pipes
// (exp2_fma2) and the rest on MUFU.  Measured on B200 at S = 16K and 32K: 0 is fastest for
// this kernel (the softmax warps are issue-bound, and the polynomial costs more issue slots
// than the MUFU cycles it saves), so the knob stays at 0.
#ifndef RA_FWD_EXP2_FMA_PER4
#define RA_FWD_EXP2_FMA_PER4 0
#endif
constexpr uint32_t TMEM_COLS = 512;

template <int HD>
struct Layout {
  static_assert(HD == 64 || HD == 128, "head dim");
  static constexpr int SUB = HD / 64;                  // 128-byte-swizzled column blocks
  static constexpr int SUB_BYTES = 128 * 128;          // 128 rows x 128 B
  static constexpr int TILE_BYTES = SUB * SUB_BYTES;   // one 128-row tile of Q, K or V
  static constexpr int Q_OFF = 0;
  static constexpr int KV_OFF = Q_OFF + NQ * TILE_BYTES;
  static constexpr int BAR_OFF = KV_OFF + NSTAGE * TILE_BYTES;
  // barrier indices
  static constexpr int B_Q_FULL = 0, B_Q_EMPTY = 1, B_KV_FULL = 2, B_KV_EMPTY = B_KV_FULL + NSTAGE,
                       B_S_FULL = B_KV_EMPTY + NSTAGE, B_P_READY = B_S_FULL + NQ, B_O_FINAL = B_P_READY + NQ,
                       B_DRAIN = B_O_FINAL + NQ, B_WQ_FULL = B_DRAIN + 1, B_WQ_EMPTY = B_WQ_FULL + 2,
                       NUM_BARS = B_WQ_EMPTY + 2;
  static constexpr uint32_t WQ_CONSUMERS = 1 + 8;   // MMA thread + one arrival per softmax warp
  static constexpr int MISC_OFF = BAR_OFF + NUM_BARS * 8;   // TMEM base, abort flag, item ring[2]
  static constexpr int BYTES = MISC_OFF + 16;
  static constexpr int ALLOC = BYTES + 1024;           // room to align the base to 1024 B
  // TMEM columns of S_t (P_t aliases its first 64) and of O_t.
  __host__ __device__ static constexpr uint32_t s_col(int t) { return 128u * t; }
  __host__ __device__ static constexpr uint32_t o_col(int t) { return 256u + uint32_t(HD) * t; }
};

struct Params {
  int BH, S, D, causal;
  int n_pairs;        // ceil(S / ROWS)
  int n_parts;        // pieces each pair's visit order is cut into (1: no split)
  int n_items;        // BH * n_pairs * n_parts
  int hgroup;         // heads whose items are interleaved (L2 reuse of K, V)
  int work_slot;      // this launch's work counter
  float scale_log2;   // softmax scale * log2(e)
  __nv_bfloat16* o;   // [BH][S][HD]                  (n_parts == 1)
  float* lse;         // [BH][S]
  float* o_part;      // [n_parts][BH][S][HD] fp32, normalised per part   (n_parts > 1)
  float* lse_part;    // [n_parts][BH][S], natural log, -inf for a row that sees no key of the part
};

// Work item w -> (bh, pair, part).  Heads are taken in groups of p.hgroup (all heads by
// default); inside a group items go pair by pair, causal: the last query tiles (longest
// items) first, so the CTAs that fetch items dynamically finish together; the parts of one
// pair are adjacent.
template <bool SPLIT>
__device__ __forceinline__ void item_coords(int w, const Params& p, int& bh, int& pair, int& part) {
  const int n_parts = SPLIT ? p.n_parts : 1;
  const int per_group = p.hgroup * p.n_pairs * n_parts;
  const int g = w / per_group;
  const int gsize = min(p.hgroup, p.BH - g * p.hgroup);
  const int idx = w - g * per_group;
  const int rank = idx / gsize;
  bh = g * p.hgroup + (idx - rank * gsize);
  const int pair_rank = SPLIT ? rank / n_parts : rank;
  part = rank - pair_rank * n_parts;
  pair = p.causal ? (p.n_pairs - 1 - pair_rank) : pair_rank;
}

__device__ __forceinline__ void advance(int& stage, uint32_t& phase) {
  if (++stage == NSTAGE) {
    stage = 0;
    phase ^= 1u;
  }
}

// ------------------------------------------------------------------ producer (1 thread)
template <int HD, bool SPLIT>
__device__ void producer(const CUtensorMap* tm_q, const CUtensorMap* tm_k, const CUtensorMap* tm_v,
                         const Params& p, uint32_t sbase, volatile int* wq, volatile int* abort_flag) {
  using L = Layout<HD>;
  const uint32_t bars = sbase + L::BAR_OFF;
  auto bar = [&](int i) { return bars + 8u * i; };
  int stage = 0;
  uint32_t phase = 0, q_phase = 0;
  uint32_t issued = 0, issued_parity = 0;   // per stage: ever armed / parity of last arm
  int q_issued = 0;
  uint32_t q_parity = 0;
  bool ok = true;
  ItemRing ring{bar(L::B_WQ_FULL), bar(L::B_WQ_EMPTY), wq};
  int w = work_fetch(p.work_slot);
  for (;;) {
    if (!ring.push(w, abort_flag)) { ok = false; break; }
    if (w >= p.n_items) break;
    const int w_next = work_fetch(p.work_slot);   // in flight while this item's loads issue
    int bh, pair, part;
    item_coords<SPLIT>(w, p, bh, pair, part);
    const int q0 = pair * ROWS;
    RingTiles it;
    it.init(p.S, p.D, p.causal, q0, ROWS, BN);
    if (SPLIT && it.restrict_to(part, p.n_parts) == 0) {   // empty piece: nothing to load
      w = w_next;
      continue;
    }
    if (!mbar_wait(bar(L::B_Q_EMPTY), q_phase ^ 1u, abort_flag)) { ok = false; break; }
    mbar_arrive_expect_tx(bar(L::B_Q_FULL), NQ * L::TILE_BYTES);
#pragma unroll
    for (int t = 0; t < NQ; ++t)
#pragma unroll
      for (int sb = 0; sb < L::SUB; ++sb)
        tma_load_3d(tm_q, sbase + L::Q_OFF + t * L::TILE_BYTES + sb * L::SUB_BYTES, bar(L::B_Q_FULL), sb * 64,
                    q0 + t * BM, bh);
    q_issued = 1;
    q_parity = q_phase;
    q_phase ^= 1u;

    for (int kt = (SPLIT ? it.next_in_part() : it.next()); kt >= 0; kt = (SPLIT ? it.next_in_part() : it.next())) {
#pragma unroll
      for (int kv = 0; kv < 2; ++kv) {
        if (!mbar_wait(bar(L::B_KV_EMPTY + stage), phase ^ 1u, abort_flag)) { ok = false; break; }
        mbar_arrive_expect_tx(bar(L::B_KV_FULL + stage), L::TILE_BYTES);
        const CUtensorMap* tm = kv ? tm_v : tm_k;
#pragma unroll
        for (int sb = 0; sb < L::SUB; ++sb)
          tma_load_3d(tm, sbase + L::KV_OFF + stage * L::TILE_BYTES + sb * L::SUB_BYTES, bar(L::B_KV_FULL + stage),
                      sb * 64, kt * BN, bh);
        issued |= 1u << stage;
        issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
        advance(stage, phase);
      }
      if (!ok) break;
    }
    if (!ok) break;
    w = w_next;
  }
  work_done(p.work_slot);
  if (!ok) {  // let every copy this CTA started land before the CTA can exit
    for (int s = 0; s < NSTAGE; ++s)
      if (issued & (1u << s)) drain_wait(bar(L::B_KV_FULL + s), (issued_parity >> s) & 1u);
    if (q_issued) drain_wait(bar(L::B_Q_FULL), q_parity);
  }
}

// ------------------------------------------------------------------ MMA issuer (1 thread)
template <int HD>
__device__ __forceinline__ void issue_qk(uint32_t sbase, uint32_t tmem, int t, int kstage) {
  using L = Layout<HD>;
  constexpr uint32_t IDESC = idesc_bf16_f32(BM, BN, 0, 0);  // A = Q (K-major), B = K (K-major)
  const uint32_t qa = sbase + L::Q_OFF + t * L::TILE_BYTES;
  const uint32_t ka = sbase + L::KV_OFF + kstage * L::TILE_BYTES;
#pragma unroll
  for (int kk = 0; kk < HD / 16; ++kk) {
    const uint32_t off = (kk >> 2) * L::SUB_BYTES + (kk & 3) * 32;
    umma_ss(tmem + L::s_col(t), sdesc_sw128(qa + off, 16, 1024), sdesc_sw128(ka + off, 16, 1024), IDESC,
            kk > 0 ? 1u : 0u);
  }
}

template <int HD>
__device__ __forceinline__ void issue_pv(uint32_t sbase, uint32_t tmem, int t, int vstage, bool accumulate) {
  using L = Layout<HD>;
  constexpr uint32_t IDESC = idesc_bf16_f32(BM, HD, 0, 1);  // A = P (TMEM), B = V (MN-major)
  const uint32_t va = sbase + L::KV_OFF + vstage * L::TILE_BYTES;
#pragma unroll
  for (int kk = 0; kk < BN / 16; ++kk) {
    // 16 keys per step: two 8-row groups of the V tile (1024 B each); the two 64-column
    // halves of V (HD = 128) are L::SUB_BYTES apart.
    umma_ts(tmem + L::o_col(t), tmem + L::s_col(t) + kk * 8, sdesc_sw128(va + kk * 2048, L::SUB_BYTES, 1024),
            IDESC, (accumulate || kk > 0) ? 1u : 0u);
  }
}

template <int HD, bool SPLIT>
__device__ void mma_issuer(const Params& p, uint32_t sbase, uint32_t tmem, volatile int* wq, volatile int* abort_flag) {
  using L = Layout<HD>;
  const uint32_t bars = sbase + L::BAR_OFF;
  auto bar = [&](int i) { return bars + 8u * i; };
  int stage = 0;
  uint32_t phase = 0, q_phase = 0;
  uint32_t p_phase[NQ] = {0, 0};
  bool ok = true;
  ItemRing ring{bar(L::B_WQ_FULL), bar(L::B_WQ_EMPTY), wq};
  for (;;) {
    int w;
    if (!ring.pop(w, abort_flag)) { ok = false; break; }
    if (w >= p.n_items) break;
    int bh, pair, part;
    item_coords<SPLIT>(w, p, bh, pair, part);
    RingTiles it;
    it.init(p.S, p.D, p.causal, pair * ROWS, ROWS, BN);
    if (SPLIT && it.restrict_to(part, p.n_parts) == 0) continue;   // empty piece
    if (!mbar_wait(bar(L::B_Q_FULL), q_phase, abort_flag)) { ok = false; break; }
    q_phase ^= 1u;
    tc_fence_after();
    int vprev = 0, n = 0;
    for (int kt = (SPLIT ? it.next_in_part() : it.next()); kt >= 0; kt = (SPLIT ? it.next_in_part() : it.next()), ++n) {
      const int ks = stage;
      if (!mbar_wait(bar(L::B_KV_FULL + ks), phase, abort_flag)) { ok = false; break; }
      advance(stage, phase);
      tc_fence_after();
#pragma unroll
      for (int t = 0; t < NQ; ++t) {
        if (n > 0) {
          if (!mbar_wait(bar(L::B_P_READY + t), p_phase[t], abort_flag)) { ok = false; break; }
          p_phase[t] ^= 1u;
          tc_fence_after();
          issue_pv<HD>(sbase, tmem, t, vprev, n > 1);
          if (t == NQ - 1) tc_commit(bar(L::B_KV_EMPTY + vprev));
        }
        issue_qk<HD>(sbase, tmem, t, ks);
        tc_commit(bar(L::B_S_FULL + t));
      }
      if (!ok) break;
      tc_commit(bar(L::B_KV_EMPTY + ks));
      const int vs = stage;
      if (!mbar_wait(bar(L::B_KV_FULL + vs), phase, abort_flag)) { ok = false; break; }
      advance(stage, phase);
      tc_fence_after();
      vprev = vs;
    }
    if (!ok) break;
    tc_commit(bar(L::B_Q_EMPTY));  // Q tiles no longer read once these MMAs complete
#pragma unroll
    for (int t = 0; t < NQ; ++t) {
      if (!mbar_wait(bar(L::B_P_READY + t), p_phase[t], abort_flag)) { ok = false; break; }
      p_phase[t] ^= 1u;
      tc_fence_after();
      issue_pv<HD>(sbase, tmem, t, vprev, n > 1);
      tc_commit(bar(L::B_O_FINAL + t));
    }
    if (!ok) break;
    tc_commit(bar(L::B_KV_EMPTY + vprev));
  }
  // Wait until every MMA this thread issued has completed before TMEM is released.
  tc_commit(bar(L::B_DRAIN));
  drain_wait(bar(L::B_DRAIN), 0);
}

// ------------------------------------------------------------------ softmax (128 threads)
template <int HD, bool SPLIT>
__device__ void softmax_wg(int t, const Params& p, uint32_t sbase, uint32_t tmem, volatile int* wq,
                           volatile int* abort_flag) {
  using L = Layout<HD>;
  const uint32_t bars = sbase + L::BAR_OFF;
  auto bar = [&](int i) { return bars + 8u * i; };
  const int lane = threadIdx.x & 31;
  const int quarter = (threadIdx.x >> 5) & 3;     // TMEM lanes 32*quarter .. +31
  const int row = quarter * 32 + lane;            // row within the query tile
  const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
  const uint32_t tS = lane_base + L::s_col(t);
  const uint32_t tO = lane_base + L::o_col(t);
  const float sl2 = p.scale_log2;
  uint32_t s_phase = 0, o_phase = 0;

  ItemRing ring{bar(L::B_WQ_FULL), bar(L::B_WQ_EMPTY), wq};
  for (;;) {
    int w;
    if (!ring.pop_warp(w, abort_flag)) return;
    if (w >= p.n_items) break;
    int bh, pair, part;
    item_coords<SPLIT>(w, p, bh, pair, part);
    const int q_tile0 = pair * ROWS + t * BM;
    const int q_row = q_tile0 + row;
    const int vis_end = (p.causal && q_row + 1 < p.S) ? q_row + 1 : p.S;  // keys [0, vis_end) visible
    const bool row_ok = q_row < p.S;
    float m_ref = -INFINITY;   // exponent reference (log2 units), raised lazily
    float l = 0.f;
    RingTiles it;
    it.init(p.S, p.D, p.causal, pair * ROWS, ROWS, BN);
    if (SPLIT && it.restrict_to(part, p.n_parts) == 0) {   // empty piece: O = 0, lse = -inf
      if (row_ok) {
        const size_t prow = (static_cast<size_t>(part) * p.BH + bh) * p.S + q_row;
        float4* dst = reinterpret_cast<float4*>(p.o_part + prow * HD);
#pragma unroll
        for (int i = 0; i < HD / 4; ++i) dst[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        p.lse_part[prow] = -INFINITY;
      }
      continue;
    }
    int n = 0;
    for (int kt = (SPLIT ? it.next_in_part() : it.next()); kt >= 0; kt = (SPLIT ? it.next_in_part() : it.next()), ++n) {
      // all 32 lanes must agree before the warp-collective TMEM loads below
      if (!__all_sync(0xffffffffu, mbar_wait(bar(L::B_S_FULL + t), s_phase, abort_flag))) return;
      s_phase ^= 1u;
      tc_fence_after();
      uint32_t s[BN];
#pragma unroll
      for (int c = 0; c < BN / 32; ++c) tmem_ld32(tS + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&s[32 * c]));
      tmem_ld_wait();

      const int k0 = kt * BN;
      const bool masked_tile = (k0 + BN > p.S) || (p.causal && k0 + BN - 1 > q_tile0);
      if (masked_tile) {
        const int lim = vis_end - k0;
#pragma unroll
        for (int c = 0; c < BN; ++c)
          if (c >= lim) s[c] = __float_as_uint(-INFINITY);
      }
      float mx;
      {  // row max: four independent chains of three-input maxima
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int c = 0; c < BN; c += 8)
#pragma unroll
          for (int j = 0; j < 4; ++j)
            m4[j] = fmax3(m4[j], __uint_as_float(s[c + 2 * j]), __uint_as_float(s[c + 2 * j + 1]));
        mx = fmax3(m4[0], m4[1], fmaxf(m4[2], m4[3]));
      }
      const float m_tile = mx * sl2;
      const float m_new = fmaxf(m_ref, m_tile);
      const bool raise = m_new > m_ref + RESCALE_LOG2;   // false while nothing is visible
      const float alpha = raise ? (m_ref == -INFINITY ? 0.f : ex2_approx(m_ref - m_new)) : 1.f;
      if (n > 0 && __any_sync(0xffffffffu, raise)) {
        // O_t (complete: the PV before this tile's S finished before S_full fired)
#pragma unroll 1
        for (int c = 0; c < HD / 16; ++c) {
          uint32_t o[16];
          tmem_ld16(tO + 16 * c, o);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st16(tO + 16 * c, o);
        }
        tmem_st_wait();
      }
      if (raise) {
        l *= alpha;
        m_ref = m_new;
      }
      const float neg_ref = (m_ref == -INFINITY) ? 0.f : -m_ref;
      const float2 sl2x2 = make_float2(sl2, sl2), nref2 = make_float2(neg_ref, neg_ref);
      float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll
      for (int h = 0; h < 2; ++h) {   // two halves of 64 keys -> 32 packed columns each
        uint32_t pk[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const float2 x = __ffma2_rn(make_float2(__uint_as_float(s[64 * h + 2 * c]),
                                                  __uint_as_float(s[64 * h + 2 * c + 1])), sl2x2, nref2);
          float2 pp;
          if ((c & 3) < RA_FWD_EXP2_FMA_PER4) {
            pp = exp2_fma2(x);
          } else {
            pp.x = ex2_approx(x.x);
            pp.y = ex2_approx(x.y);
          }
          if (c & 1)
            acc1 = __fadd2_rn(acc1, pp);
          else
            acc0 = __fadd2_rn(acc0, pp);
          pk[c] = pack_bf16x2(pp.x, pp.y);
        }
        tmem_st32(tS + 32 * h, pk);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(L::B_P_READY + t));   // the row sum is not needed by the MMA
      l += (acc0.x + acc0.y) + (acc1.x + acc1.y);
    }
    // epilogue: O = O_acc / l (bf16), LSE = (m_ref + log2 l) * ln 2
    if (!__all_sync(0xffffffffu, mbar_wait(bar(L::B_O_FINAL + t), o_phase, abort_flag))) return;
    o_phase ^= 1u;
    tc_fence_after();
    const float inv_l = l > 0.f ? 1.f / l : 0.f;
    const float lse_row = l > 0.f ? (m_ref + log2f(l)) * 0.69314718055994531f : -INFINITY;
    if (SPLIT) {   // normalised fp32 partial of this piece, merged through its lse
      const size_t prow = (static_cast<size_t>(part) * p.BH + bh) * p.S + q_row;
      float* orow = p.o_part + prow * HD;
#pragma unroll
      for (int c = 0; c < HD / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tO + 32 * c, o);
        tmem_ld_wait();
        if (row_ok) {
          float4* dst = reinterpret_cast<float4*>(orow + 32 * c);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            dst[i] = make_float4(__uint_as_float(o[4 * i]) * inv_l, __uint_as_float(o[4 * i + 1]) * inv_l,
                                 __uint_as_float(o[4 * i + 2]) * inv_l, __uint_as_float(o[4 * i + 3]) * inv_l);
        }
      }
      if (row_ok) p.lse_part[prow] = lse_row;
      continue;
    }
    __nv_bfloat16* orow = p.o + (static_cast<size_t>(bh) * p.S + q_row) * HD;
#pragma unroll
    for (int c = 0; c < HD / 32; ++c) {
      uint32_t o[32];
      tmem_ld32(tO + 32 * c, o);
      tmem_ld_wait();
      uint32_t w16[16];
#pragma unroll
      for (int i = 0; i < 16; ++i)
        w16[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv_l, __uint_as_float(o[2 * i + 1]) * inv_l);
      if (row_ok) {
        uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
        for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w16[4 * i], w16[4 * i + 1], w16[4 * i + 2], w16[4 * i + 3]);
      }
    }
    if (row_ok) p.lse[static_cast<size_t>(bh) * p.S + q_row] = lse_row;
  }
}

// ------------------------------------------------------------------ kernel
template <int HD, bool SPLIT>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const Params p) {
  using L = Layout<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 4);
  volatile int* wq = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 8);
  const int warp = threadIdx.x >> 5;

  if (threadIdx.x == 0) {
    const uint32_t bars = sbase + L::BAR_OFF;
    for (int i = 0; i < L::NUM_BARS; ++i) {
      const bool p_ready = (i >= L::B_P_READY && i < L::B_P_READY + NQ);
      const bool wq_empty = (i >= L::B_WQ_EMPTY && i < L::B_WQ_EMPTY + 2);
      mbar_init(bars + 8u * i, p_ready ? BM : (wq_empty ? L::WQ_CONSUMERS : 1));
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
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp >= 8) {
    regs_lower<REGS_OTHER>();
    if (warp == WARP_TMA) {
      if ((threadIdx.x & 31) == 0) producer<HD, SPLIT>(&tm_q, &tm_k, &tm_v, p, sbase, wq, abort_flag);
      __syncwarp();
    } else if (warp == WARP_MMA) {
      if ((threadIdx.x & 31) == 0) mma_issuer<HD, SPLIT>(p, sbase, tmem, wq, abort_flag);
      __syncwarp();
    }
  } else {
    regs_raise<REGS_SOFTMAX>();
    softmax_wg<HD, SPLIT>(warp >> 2, p, sbase, tmem, wq, abort_flag);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == WARP_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace fwd
}  // namespace ra
