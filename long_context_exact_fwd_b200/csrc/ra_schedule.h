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
};

}  // namespace ra
