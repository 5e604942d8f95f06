// Ring schedule at tile granularity, usable from host and device code.
//
// Page "精读笔记 · Ring Attention with Blockwise Transformers for Near-Infinite Context",
// §3.2 and the 4-device walk-through of §3.5: the sequence is cut into D blocks of
// c = S / D tokens; at ring step t the position holding query block r works on key/value
// block (r - t) mod D, step 0 being its own block.  On one GPU the positions are virtual,
// so the schedule only fixes the order in which a query tile visits key/value tiles.
//
// A query tile [q0, q0 + rows) belongs to the block r of its first row.  For t = 0..D-1
// it visits, ascending, the key tiles of `kt_size` keys whose first key lies in block
// (r - t) mod D.  Under the causal mask, tiles whose first key lies after the tile's last
// query row hold no visible key and are dropped (for blocks j > r this drops the whole
// block when c is a multiple of the tile size).  Every other key tile is visited exactly
// once, whatever c is.
#pragma once

#if defined(__CUDACC__)
#define RA_HD __host__ __device__ __forceinline__
#else
#define RA_HD inline
#endif

namespace ra {

struct RingTiles {
  int D, c, kt_size, r, t, kt, kt_end, kt_limit;

  RA_HD static int cdiv(long long a, long long b) { return static_cast<int>((a + b - 1) / b); }

  RA_HD void init(int S, int D_, int causal, int q0, int rows, int kt_size_) {
    D = D_;
    c = S / D_;
    kt_size = kt_size_;
    r = q0 / c;
    t = 0;
    const int n_tiles = cdiv(S, kt_size);
    const int q_last = (q0 + rows < S ? q0 + rows : S) - 1;
    kt_limit = causal ? (q_last / kt_size + 1) : n_tiles;
    set_block();
  }

  RA_HD void set_block() {
    const int j = ((r - t) % D + D) % D;
    kt = cdiv(static_cast<long long>(j) * c, kt_size);
    const int e = cdiv(static_cast<long long>(j + 1) * c, kt_size);
    kt_end = e < kt_limit ? e : kt_limit;
  }

  // Next key tile index in visit order, or -1 when the schedule is exhausted.
  RA_HD int next() {
    while (t < D) {
      if (kt < kt_end) return kt++;
      if (++t < D) set_block();
    }
    return -1;
  }

  // Number of key tiles the whole visit order holds (call right after init; leaves the
  // iterator where init put it).
  RA_HD int count() const {
    int n = 0;
    for (int u = 0; u < D; ++u) {
      const int j = ((r - u) % D + D) % D;
      const int a = cdiv(static_cast<long long>(j) * c, kt_size);
      const int e0 = cdiv(static_cast<long long>(j + 1) * c, kt_size);
      const int e = e0 < kt_limit ? e0 : kt_limit;
      if (e > a) n += e - a;
    }
    return n;
  }

  // Restrict the iterator to part `part` of `n_parts` contiguous, near-equal pieces of the
  // visit order (pieces [n*part/n_parts, n*(part+1)/n_parts) of the n tiles); returns the
  // number of tiles in the piece (0 when n < n_parts leaves it empty).  Call right after init.
  RA_HD int restrict_to(int part, int n_parts) {
    const int n = count();
    const int lo = static_cast<int>(static_cast<long long>(n) * part / n_parts);
    const int hi = static_cast<int>(static_cast<long long>(n) * (part + 1) / n_parts);
    for (int i = 0; i < lo; ++i) next();
    left = hi - lo;
    return left;
  }

  // next() bounded by restrict_to's piece (call instead of next() after restrict_to).
  RA_HD int next_in_part() {
    if (left <= 0) return -1;
    --left;
    return next();
  }

  int left = 1 << 30;   // tiles next_in_part may still return (unbounded until restrict_to)
};

// The backward's view of the same ring: key/value block j sits at ring position
// (j + t) mod D at step t, so a key tile [k0, k0 + 128) visits, for t = 0..D-1, the query
// tiles of `qt_size` rows whose first row lies in block (j + t) mod D, ascending; under the
// causal mask, query tiles whose last row precedes k0 see none of its keys and are dropped.
struct RingQTiles {
  int D, c, qt_size, t, j, qt, qt_end, qt_min, n_qt;

  RA_HD void init(int S, int D_, int causal, int k0, int qt_size_) {
    D = D_;
    c = S / D_;
    qt_size = qt_size_;
    j = k0 / c;
    t = 0;
    n_qt = RingTiles::cdiv(S, qt_size);
    qt_min = causal ? k0 / qt_size : 0;   // tile i ends at row qt_size * (i + 1) - 1
    set_block();
  }

  RA_HD void set_block() {
    const int p = (j + t) % D;
    const int a = RingTiles::cdiv(static_cast<long long>(p) * c, qt_size);
    const int b = RingTiles::cdiv(static_cast<long long>(p + 1) * c, qt_size);
    qt = a > qt_min ? a : qt_min;
    qt_end = b < n_qt ? b : n_qt;
  }

  // Next query tile index in visit order, or -1.
  RA_HD int next() {
    while (t < D) {
      if (qt < qt_end) return qt++;
      if (++t < D) set_block();
    }
    return -1;
  }
};

}  // namespace ra
