/*
 * ring_attn.h -- C ABI of libringattn.so: exact ring attention on one NVIDIA B200 (sm_100a).
 *
 * What is computed (page: "精读笔记 · Ring Attention with Blockwise Transformers for
 * Near-Infinite Context", §3.1-§3.5; page: "Ring Attention 与序列并行", conceptual
 * pseudocode).  The S tokens of every (batch, head) are cut into D ring blocks of
 * c = S / D tokens.  Query block r visits the key/value blocks in ring order -- at ring
 * step t it works on block (r - t) mod D, step 0 being its own block -- and folds each
 * block into a running max, running sum and rescaled accumulator (online softmax).  The
 * result equals plain softmax(Q K^T * scale + mask) V with no approximation.  On one GPU
 * the D positions are virtual: the same kernel processes all of them; no data moves
 * between devices.
 *
 * Conventions shared by every entry point
 *   Layout     all per-token tensors are dense row-major [B][H][S][Dh] (Dh contiguous);
 *              LSE and the other per-row statistics are [B][H][S] float32.
 *   Pointers   device pointers (cudaMalloc / torch CUDA memory) unless stated; tensors
 *              read by TMA (q, k, v and the backward inputs) must be 16-byte aligned.
 *              The caller owns every buffer; the library never allocates or frees device
 *              memory and never synchronises, except ring_attn_device_status.
 *   Stream     `stream` is a cudaStream_t (NULL = legacy default stream); all work is
 *              enqueued on it.  Calls return as soon as the work is enqueued.
 *   Mask       causal != 0 selects the autoregressive mask on global positions: key j is
 *              visible to query i iff j <= i.  The pages never state a mask; this is the
 *              standard reading.  causal == 0 lets every query see every key.
 *   Scale      scores are q.k * scale with scale = 1/sqrt(Dh) unless an _ex call passes
 *              scale > 0.
 *   LSE        natural log of sum_j exp(score_ij) over visible keys, float32.
 *   Errors     every call returns RA_OK (0) or one of the RA_ERR_* codes below and never
 *              throws; argument errors are detected before anything is enqueued.  A
 *              device-side fault surfaces at the caller's next synchronisation.  A kernel
 *              whose internal bounded wait expired leaves RA_ERR_TIMEOUT in the device
 *              status word, read by ring_attn_device_status.
 */
#ifndef RING_ATTN_H_
#define RING_ATTN_H_

#include <stddef.h>

#if defined(__GNUC__)
#define RA_API __attribute__((visibility("default")))
#else
#define RA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

enum {
  RA_OK = 0,
  RA_ERR_ARG = 1,         /* null pointer, non-positive size, unknown dtype            */
  RA_ERR_SHAPE = 2,       /* S % D != 0, unsupported Dh, or a size that overflows       */
  RA_ERR_ALIGN = 3,       /* a TMA-read pointer is not 16-byte aligned                 */
  RA_ERR_WORKSPACE = 4,   /* workspace null or smaller than required                   */
  RA_ERR_CUDA = 5,        /* a CUDA runtime or driver call failed                      */
  RA_ERR_TIMEOUT = 6,     /* a kernel gave up on a bounded internal wait               */
  RA_ERR_DEVICE = 7       /* the current device is not compute capability 10.0         */
};

typedef enum { RA_BF16 = 0, RA_F32 = 1 } ra_dtype;

/* A cudaStream_t, passed as an opaque pointer so this header needs no CUDA headers. */
typedef void* ra_stream;

/*
 * ring_attn_fwd -- forward pass, bf16 inputs (page "精读笔记 ...", §3.1 and §3.5 Algorithm 1).
 *   q, k, v  [B][H][S][Dh] bf16, read only, 16-byte aligned.
 *   o        [B][H][S][Dh] bf16, written: O = softmax(q k^T / sqrt(Dh) + mask) v, fp32
 *            accumulated and rounded to nearest even once.
 *   lse      [B][H][S] float32, written: the row log-sum-exp (natural log).
 *   B, H, S  >= 1.  S need not be a multiple of the kernel's 128-row tiles.
 *   Dh       head dimension: 64 or 128 (else RA_ERR_SHAPE).
 *   D        number of ring blocks, 1 <= D <= S and S % D == 0 (the pages' even split,
 *            "limitations" paragraph of the close reading), else RA_ERR_SHAPE.
 *   causal   0 or 1 (see Mask above).
 * The result does not depend on D (order independence, §3.1); D fixes the order in which
 * each query tile visits the key/value tiles.
 */
RA_API int ring_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int S,
                  int Dh, int D, int causal, ra_stream stream);

/*
 * ring_attn_fwd_ex -- forward pass with an explicit input dtype and scale.
 *   dtype RA_BF16: as ring_attn_fwd (o is bf16).
 *   dtype RA_F32 : q, k, v and o are float32; scores, exponentials and the accumulator are
 *                  float32 on CUDA cores (no tensor-core rounding), any Dh in 1..256.
 *   scale > 0 overrides 1/sqrt(Dh); scale <= 0 keeps the default.
 */
RA_API int ring_attn_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int S,
                     int Dh, int D, int causal, ra_dtype dtype, float scale, ra_stream stream);

/* Largest n_parts ring_attn_fwd_split accepts. */
#define RA_MAX_FWD_PARTS 16

/*
 * ring_attn_fwd_split_workspace_size -- bytes of device workspace ring_attn_fwd_split needs
 * for n_parts pieces: n_parts float32 partial outputs [B][H][S][Dh] followed by n_parts
 * float32 partial log-sum-exps [B][H][S] (that region rounded up to 256 bytes per part).
 * Returns 0 for invalid sizes.
 */
RA_API size_t ring_attn_fwd_split_workspace_size(int B, int H, int S, int Dh, int n_parts);

/*
 * ring_attn_fwd_split -- forward pass with each query block's ring cut into pieces that run
 * on different SMs, then merged (page "精读笔记 ...", §3.1: partial results over disjoint
 * sets of key/value blocks, combined in any order through their statistics; page
 * "RingAttention large-context attention", 架构与算法: partial outputs aggregated into the
 * final output).  For few heads and long sequences the longest query blocks otherwise keep a
 * handful of SMs busy after the rest have finished.
 *   q, k, v, o, lse, B, H, S, Dh, D, causal  as ring_attn_fwd (Dh 64 or 128).
 *   n_parts   1..RA_MAX_FWD_PARTS.  Each 256-row query pair's key tiles, in ring order, are
 *             cut into n_parts contiguous pieces of near-equal tile count; piece p is one
 *             work item.  A pair with fewer tiles than n_parts leaves some pieces empty
 *             (lse -inf, weight 0 in the merge).  n_parts = 1 is ring_attn_fwd exactly and
 *             needs no workspace.
 *   workspace device memory of at least ring_attn_fwd_split_workspace_size(...) bytes,
 *             256-byte aligned, owned by the caller; its contents on entry do not matter and
 *             on return hold the partials (o_part, lse_part) for inspection.
 * Two launches on `stream`: the forward kernel writing the partials, then ring_attn_merge.
 * Errors: RA_ERR_ARG (null pointer, n_parts out of range), RA_ERR_SHAPE, RA_ERR_ALIGN (inputs
 * not 16-byte or workspace not 256-byte aligned), RA_ERR_WORKSPACE (missing or too small),
 * RA_ERR_CUDA.
 */
RA_API int ring_attn_fwd_split(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int S,
                               int Dh, int D, int causal, int n_parts, void* workspace, size_t workspace_bytes,
                               ra_stream stream);

/*
 * ring_attn_fwd_partial -- ring_attn_fwd with a float32 output, for results that are merged
 * afterwards (page "精读笔记 ...", §3.1: the output over one set of key/value blocks, kept
 * with its log-sum-exp so that it can be combined with others; the multi-GPU ring merges one
 * such partial per ring step).
 *   q, k, v, B, H, S, Dh, D, causal  as ring_attn_fwd (bf16, Dh 64 or 128).
 *   o_part    [B][H][S][Dh] float32, written: the normalised output O (not rounded to bf16).
 *   lse_part  [B][H][S] float32, written: natural-log LSE of each row.
 * Together they are one part of ring_attn_merge's input.  One launch on `stream`.
 * Errors: RA_ERR_ARG (null pointer), RA_ERR_SHAPE, RA_ERR_ALIGN (q, k, v or o_part not 16-byte
 * aligned), RA_ERR_CUDA.
 */
RA_API int ring_attn_fwd_partial(const void* q, const void* k, const void* v, float* o_part, float* lse_part, int B,
                                 int H, int S, int Dh, int D, int causal, ra_stream stream);

/*
 * ring_attn_bwd_workspace_size -- bytes of device workspace ring_attn_bwd needs: a float32
 * dQ accumulator [B][H][S][Dh] and two float32 row statistics (Delta = rowsum(dO * O) and
 * lse * log2(e)) of [B][H][S_pad] with S_pad = S rounded up to 128, each region 256-byte
 * aligned.  Returns 0 for invalid sizes.
 */
RA_API size_t ring_attn_bwd_workspace_size(int B, int H, int S, int Dh);

/*
 * ring_attn_bwd -- backward pass of ring_attn_fwd (bf16).  The pages state that training runs
 * through the same blockwise ring structure but give no formulas; this is the analytic
 * softmax gradient, with P recomputed from the saved LSE:
 *   P = exp(q k^T * scale - lse), dV = P^T dO, dP = dO V^T, Delta = rowsum(dO * O),
 *   dS = P * (dP - Delta), dQ = scale * dS K, dK = scale * dS^T Q.
 *   q, k, v, o, dO : [B][H][S][Dh] bf16, read only, 16-byte aligned (o from ring_attn_fwd).
 *   lse            : [B][H][S] float32 from ring_attn_fwd.
 *   dq, dk, dv     : [B][H][S][Dh] bf16, written (fully overwritten).
 *   Dh             : 64 or 128 (else RA_ERR_SHAPE).
 *   workspace      : >= ring_attn_bwd_workspace_size(B, H, S, Dh) bytes of device memory,
 *                    256-byte aligned; its contents on entry are ignored (it is cleared
 *                    on the stream) and undefined on return.
 *   Other arguments as ring_attn_fwd.  Each key/value tile visits the query tiles that
 *   can see it, in ring order.  Three launches on `stream` (Delta preprocess, main kernel, dQ
 *   conversion).  Errors: RA_ERR_ARG (null pointer, non-positive size), RA_ERR_SHAPE,
 *   RA_ERR_ALIGN, RA_ERR_WORKSPACE (null, not 256-byte aligned or too small), RA_ERR_CUDA.
 */
RA_API int ring_attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
                  void* dq, void* dk, void* dv, int B, int H, int S, int Dh, int D, int causal, void* workspace,
                  size_t workspace_bytes, ra_stream stream);

/*
 * ring_attn_bwd_ex -- ring_attn_bwd with an explicit softmax scale: the gradient of
 * ring_attn_fwd_ex called with the same scale (page "精读笔记 ...", §4.2: training runs through
 * the same blockwise ring; the scale enters P = exp(scale q k^T - lse), dQ = scale dS K and
 * dK = scale dS^T Q).  scale > 0 overrides 1/sqrt(Dh); scale <= 0 (or not finite) keeps the
 * default.  lse must come from a forward with the same scale.  Other arguments, launches and
 * errors as ring_attn_bwd.
 */
RA_API int ring_attn_bwd_ex(const void* q, const void* k, const void* v, const void* o, const float* lse,
                            const void* dO, void* dq, void* dk, void* dv, int B, int H, int S, int Dh, int D,
                            int causal, float scale, void* workspace, size_t workspace_bytes, ra_stream stream);

/*
 * ring_attn_bwd_accumulate -- ring_attn_bwd whose gradients are added, in float32, to the
 * caller's accumulators instead of written in bf16: dq32 += dQ, dk32 += dK, dv32 += dV.  For
 * gradients summed over several calls (the multi-GPU ring: dQ of a rank's queries over the
 * ring steps, dK and dV of a travelling key/value block over the ranks; page "精读笔记 ...",
 * §4.2: training runs through the same blockwise ring), rounded once by the caller at the end.
 *   q, k, v, o, lse, dO, B, H, S, Dh, D, causal, workspace  as ring_attn_bwd.
 *   dq32, dk32, dv32  [B][H][S][Dh] float32, 16-byte aligned, read and written; the caller
 *                     clears them before the first call.  Dh 64 or 128.
 * Launches as ring_attn_bwd, with the last one adding the scaled dQ instead of converting it.
 * Errors as ring_attn_bwd.
 */
RA_API int ring_attn_bwd_accumulate(const void* q, const void* k, const void* v, const void* o, const float* lse,
                                    const void* dO, float* dq32, float* dk32, float* dv32, int B, int H, int S,
                                    int Dh, int D, int causal, void* workspace, size_t workspace_bytes,
                                    ra_stream stream);

/*
 * ring_attn_bwd_noalloc -- ring_attn_bwd for callers that cannot allocate device memory.
 * The pages have no counterpart to this entry point; it exists for callers that may not call
 * cudaMalloc (or any allocator) on their path -- for example code embedded in a host
 * framework that owns every device allocation, or latency-critical code that cannot afford
 * cudaMalloc's implicit synchronisation -- and so cannot supply ring_attn_bwd's workspace.
 *   Arguments are those of ring_attn_bwd without the workspace (Dh 64 or 128).  The fp32 dQ
 *   accumulator and the per-row statistics live instead in one static device array of the
 *   library of
 *   ring_attn_bwd_noalloc_max_bytes() bytes (96 MiB), reserved on every device that loads the
 *   library until the process exits.  A problem whose ring_attn_bwd_workspace_size exceeds that
 *   size is rejected with RA_ERR_WORKSPACE before anything is enqueued.
 *   The first call on a device looks up the array's device address (cudaGetSymbolAddress) with
 *   that device current; make that first call before any stream capture.  No call allocates
 *   or frees memory.
 *   Every call on a device shares the one array, which keeps the previous call's contents; each
 *   call clears the accumulator it needs on the stream before use.  Calls whose execution
 *   overlaps on the GPU (different streams, or concurrent host threads) race on the array and
 *   give wrong gradients: serialise them.
 */
RA_API int ring_attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                                 const void* dO, void* dq, void* dk, void* dv, int B, int H, int S, int Dh, int D,
                                 int causal, ra_stream stream);

/* ring_attn_bwd_noalloc_max_bytes -- size of ring_attn_bwd_noalloc's static scratch array. */
RA_API size_t ring_attn_bwd_noalloc_max_bytes(void);

/*
 * ring_attn_ffn_workspace_size -- bytes of device workspace the blockwise feedforward needs:
 * nbuf = min(3, D) ring blocks' hidden activations, bf16 [nbuf][B][S / D][f] (block r + 1's first
 * product runs before block r's second, so that neither waits on the other's last tiles), then
 * 2 * nbuf * B * ceil((S / D) / 256) 32-bit dependency counters, each region rounded up to 256
 * bytes.  Bounded by three blocks for a given block size: the activation alive is at most three
 * blocks', never the sequence's.  Returns 0 for invalid sizes.
 */
RA_API size_t ring_attn_ffn_workspace_size(int B, int S, int D, int f);

/*
 * ring_attn_ffn_block -- the feedforward that follows attention, for ring block r only
 * (page "精读笔记 ...", §2.2: blockwise parallel transformers compute the feedforward of each
 * attention sub-layer block by block, so the largest activation is one block's hidden layer
 * -- 2bsh instead of 8bsh bytes; §3.5 Algorithm 1: per layer, each host's block goes through
 * attention and then the feedforward).  With x the block's attention output, heads side by side
 * per token (x[b, s, head * Dh + d] = o[b, head, s, d], h = H * Dh):
 *   y = gelu(x W1^T + b1) W2^T + b2,   gelu(u) = u * Phi(u) (exact form; the pages name no
 *   activation, and 8bsh bytes of bf16 activation is a hidden layer of f = 4h, the default).
 *   o         [B][H][S][Dh] bf16 attention output (ring_attn_fwd's o), read in place.
 *   B, H, S, Dh, D  as ring_attn_fwd (Dh 64 or 128); the block is tokens [r c, r c + c), c = S/D.
 *   r         ring block, 0 <= r < D (else RA_ERR_ARG).
 *   w1        [f][h] bf16 (the first layer's weight in [out][in] layout), b1 [f] float32.
 *   w2        [h][f] bf16, b2 [h] float32.
 *   f         hidden width, a positive multiple of 64.
 *   y         [B][S][h] bf16; only the block's rows are written.
 *   workspace >= ring_attn_ffn_workspace_size(B, S, D, f) bytes of device memory, 256-byte
 *             aligned: the hidden activation gelu(x W1^T + b1), rounded to bf16 (the activation
 *             the pages' memory count stores), and the dependency counters; overwritten by every
 *             call.
 * A memset of the counters and one persistent launch of CTA pairs (clusters of two CTAs on
 * neighbouring SMs) on `stream`: tcgen05 tiles of both products (bias + GELU epilogue, then bias
 * epilogue), float32 accumulation; a tile of the second product starts once the first product's
 * tiles of its rows are stored.  Pointers
 * 16-byte aligned.  Calls that overlap on the GPU must not share a workspace.  Errors:
 * RA_ERR_ARG (null pointer, f <= 0, r out of range), RA_ERR_SHAPE (S % D, Dh, f % 64, sizes),
 * RA_ERR_ALIGN, RA_ERR_WORKSPACE, RA_ERR_CUDA; RA_ERR_TIMEOUT in the device status word if a
 * bounded wait gave up.
 */
RA_API int ring_attn_ffn_block(const void* o, int B, int H, int S, int Dh, int D, int r, const void* w1,
                               const float* b1, const void* w2, const float* b2, int f, void* y, void* workspace,
                               size_t workspace_bytes, ra_stream stream);

/*
 * ring_attn_ffn_fwd -- the feedforward of every ring block r = 0 .. D-1, in that order, in one
 * persistent launch, in the order: first product of block 0, then for r = 1 .. D-1 the first
 * product of block r and the second of block r - 1, then the second of block D-1.  The
 * block-sized activation buffers of the workspace rotate (block r uses buffer r mod min(3, D)), so
 * at most three blocks' hidden activations are alive, whatever the sequence length.  Arguments and errors as
 * ring_attn_ffn_block (without r).
 */
RA_API int ring_attn_ffn_fwd(const void* o, int B, int H, int S, int Dh, int D, const void* w1, const float* b1,
                             const void* w2, const float* b2, int f, void* y, void* workspace, size_t workspace_bytes,
                             ra_stream stream);

/*
 * ring_attn_merge -- combine P normalised partial outputs through their log-sum-exp
 * (page "精读笔记 ...", §3.1: blocks may be combined in any order when their statistics are
 * combined with rescaling; page "RingAttention large-context attention", 架构与算法: the
 * partial outputs are aggregated into the final output).
 *   o_parts   [P][B][H][S][Dh] float32, partial p normalised by its own softmax sum.
 *   lse_parts [P][B][H][S] float32; -inf marks a partial with no visible key (weight 0).
 *   o         [B][H][S][Dh] bf16, written: sum_p exp(lse_p - lse) * o_p.
 *   lse       [B][H][S] float32, written: log(sum_p exp(lse_p)); -inf (and o = 0) when every
 *             partial is -inf.
 *   P >= 1, Dh % 4 == 0 and Dh <= 256, pointers 16-byte aligned.
 */
RA_API int ring_attn_merge(const float* o_parts, const float* lse_parts, int P, void* o, float* lse, int B, int H, int S,
                    int Dh, ra_stream stream);

/* ring_attn_merge_ex -- as ring_attn_merge with o of type out_dtype (RA_BF16 or RA_F32). */
RA_API int ring_attn_merge_ex(const float* o_parts, const float* lse_parts, int P, void* o, float* lse, int B, int H,
                       int S, int Dh, ra_dtype out_dtype, ra_stream stream);

/*
 * ring_attn_ring_order -- host only, no GPU needed.  Writes to blocks[0..n) the key/value
 * blocks ring position r visits, in order: block (r - t) mod D at step t = 0..D-1 (page
 * "精读笔记 ...", §3.5 4-device walk-through), dropping blocks j > r when causal.
 * Returns n (>= 1), or -RA_ERR_ARG for bad arguments or max_blocks < n.
 */
RA_API int ring_attn_ring_order(int D, int r, int causal, int* blocks, int max_blocks);

/*
 * ring_attn_visit_tiles -- host only.  The exact sequence of 128-key tiles the forward
 * kernel visits for the query tile of `tile_rows` rows starting at row q0: ring steps of
 * the query tile's block, each step's tiles (those whose first key lies in that block)
 * ascending, tiles wholly above the causal diagonal dropped.  Writes the tile indices to
 * tiles[0..n) and returns n, or -RA_ERR_ARG.
 */
RA_API int ring_attn_visit_tiles(int S, int D, int causal, int q0, int tile_rows, int* tiles, int max_tiles);

/*
 * ring_attn_bwd_visit_tiles -- host only.  The backward's query-tile visit order for the
 * key tile starting at key k0: key/value block j = k0 / (S / D) is at ring position
 * (j + t) mod D at step t, so the tile visits, for t = 0..D-1, the `tile_rows`-row query
 * tiles whose first row lies in block (j + t) mod D, ascending, dropping (causal) tiles that
 * end before k0.  Writes query tile indices to tiles[0..n) and returns n, or -RA_ERR_ARG.
 */
RA_API int ring_attn_bwd_visit_tiles(int S, int D, int causal, int k0, int tile_rows, int* tiles, int max_tiles);

/*
 * ring_attn_launch_count -- number of CUDA kernels this library has launched since it was
 * loaded (all host threads and devices); for accounting in benchmarks.
 */
RA_API unsigned long long ring_attn_launch_count(void);

/*
 * ring_attn_device_status -- synchronises `stream`, returns the device status word
 * (RA_OK or the first RA_ERR_TIMEOUT a kernel recorded) and clears it.  Returns
 * RA_ERR_CUDA if the synchronisation itself fails.
 */
RA_API int ring_attn_device_status(ra_stream stream);

/*
 * ring_attn_last_cuda_error -- diagnostics for RA_ERR_CUDA: the cudaError_t / CUresult value
 * of the last failing CUDA call made by this library on the calling host thread (0 if none),
 * and, when `site` is not NULL, a static string naming that call.
 */
RA_API int ring_attn_last_cuda_error(const char** site);

/*
 * ring_attn_wait_selftest -- exercises the bounded-wait failure path every kernel uses (no
 * counterpart on the pages): one thread waits on an mbarrier that nothing ever arrives on,
 * gives up after timeout_ns nanoseconds (0 < timeout_ns <= 1e10) and records RA_ERR_TIMEOUT in
 * the device status word, exactly as a kernel whose pipeline stalled would.  Read it back with
 * ring_attn_device_status; the context stays usable.
 */
RA_API int ring_attn_wait_selftest(long long timeout_ns, ra_stream stream);

/*
 * ring_attn_exp2_check -- numerical self-check of the two base-2 exponentials the softmax
 * kernels use (no counterpart on the pages): for i < n, y_fma[i] = the polynomial evaluation on
 * the FMA pipes (relative error <= 1.0e-4 for x in [-126, 8]) and y_mufu[i] = the hardware
 * ex2.approx unit.  x, y_fma, y_mufu are device float32 arrays of n elements.
 */
RA_API int ring_attn_exp2_check(const float* x, float* y_fma, float* y_mufu, long long n, ra_stream stream);

/* Static English text for a status code. */
RA_API const char* ring_attn_strerror(int code);

/* Library ABI version (major * 100 + minor). */
RA_API int ring_attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* RING_ATTN_H_ */
