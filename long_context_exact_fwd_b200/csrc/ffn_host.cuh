// Host side of the blockwise feedforward after attention: workspace layout, argument checks,
// tensor maps and the persistent launch of ffn_kernel, and the two C entry points.  Included once,
// at the end of ring_attn.cu (it uses that file's device info, tensor-map and status helpers).
#pragma once

// --- blockwise feedforward after attention ------------------------------------------------
namespace {

// Workspace: nbuf = min(3, D) block-sized hidden activations (bf16 [nbuf][B][c][f]) then the
// per-row-tile dependency counters ([nbuf][MT] ready, [nbuf][MT] consumed), each region 256-byte
// aligned.
struct FfnWorkspace {
  size_t z_bytes, ctr_bytes, total;
  int mt;     // row tiles of 256 per block: B * ceil(c / 256)
  int nbuf;   // block-sized hidden-activation buffers: min(3, D)
};

FfnWorkspace ffn_workspace(int B, int S, int D, int f) {
  FfnWorkspace w;
  const int c = S / D;
  w.mt = B * ((c + ra::ffn::BM - 1) / ra::ffn::BM);
  w.nbuf = D < 3 ? D : 3;
  w.z_bytes = align256(static_cast<size_t>(w.nbuf) * B * c * f * 2);
  w.ctr_bytes = align256(static_cast<size_t>(2 * w.nbuf) * w.mt * sizeof(unsigned));
  w.total = w.z_bytes + w.ctr_bytes;
  return w;
}

// Arguments shared by the two feedforward entry points; RA_OK when usable.
int ffn_check(const void* o, int B, int H, int S, int Dh, int D, const void* w1, const float* b1, const void* w2,
              const float* b2, int f, void* y, void* workspace, size_t workspace_bytes) {
  if (!o || !w1 || !b1 || !w2 || !b2 || !y) return RA_ERR_ARG;
  if (f <= 0) return RA_ERR_ARG;
  int st = check_shape(B, H, S, Dh, D);
  if (st != RA_OK) return st;
  if (Dh != 64 && Dh != 128) return RA_ERR_SHAPE;
  if (f % 64 != 0) return RA_ERR_SHAPE;
  const long long h = static_cast<long long>(H) * Dh;
  if (h > (1 << 20) || f > (1 << 24)) return RA_ERR_SHAPE;
  if (static_cast<double>(B) * S * (h > f ? h : f) > 9.0e18 / 4) return RA_ERR_SHAPE;
  for (const void* ptr : {o, w1, w2, static_cast<const void*>(b1), static_cast<const void*>(b2),
                          static_cast<const void*>(y)})
    if (!aligned16(ptr)) return RA_ERR_ALIGN;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 ||
      workspace_bytes < ffn_workspace(B, S, D, f).total)
    return RA_ERR_WORKSPACE;
  return RA_OK;
}

// Feedforward of ring blocks r0 .. r0 + nblocks - 1 in one persistent launch (after clearing the
// dependency counters on the stream).
int ffn_run(const void* o, int B, int H, int S, int Dh, int D, int r0, int nblocks, const void* w1, const float* b1,
            const void* w2, const float* b2, int f, void* y, void* workspace, cudaStream_t stream) {
  namespace rf = ra::ffn;
  int st = RA_OK;
  DevInfo* di = dev_info(&st);
  if (!di) return st;
  const FfnWorkspace ws = ffn_workspace(B, S, D, f);
  rf::Params p{};
  p.S = S;
  p.H = H;
  p.Dh = Dh;
  p.c = S / D;
  p.h = H * Dh;
  p.f = f;
  p.r0 = r0;
  p.nblocks = nblocks;
  p.mt_per_b = (p.c + rf::BM - 1) / rf::BM;
  p.MT = ws.mt;
  p.NT1 = (f + rf::BN - 1) / rf::BN;
  p.NT2 = (p.h + rf::BN - 1) / rf::BN;
  const long long per_block = static_cast<long long>(p.MT) * (p.NT1 + p.NT2);
  if (per_block * nblocks > INT_MAX) return RA_ERR_SHAPE;
  p.per_block = static_cast<int>(per_block);
  p.n_items = static_cast<int>(per_block * nblocks);
  p.nbuf = ws.nbuf;
  p.work_slot = static_cast<int>(di->next_work_slot.fetch_add(1) % ra::WORK_SLOTS);
  p.b1 = b1;
  p.b2 = b2;
  p.z = static_cast<__nv_bfloat16*>(workspace);
  p.y = static_cast<__nv_bfloat16*>(y);
  p.ready = reinterpret_cast<unsigned*>(static_cast<char*>(workspace) + ws.z_bytes);
  p.consumed = p.ready + ws.nbuf * p.MT;
  CUtensorMap mx, mw1, mz, mw2;
  // each CTA of a pair loads 128 rows of A and 128 of the tile's 256 B rows per K step
  if ((st = make_map(&mx, o, static_cast<long long>(B) * H, S, Dh, rf::HALF)) != RA_OK) return st;
  if ((st = make_map(&mw1, w1, 1, f, p.h, rf::HALF)) != RA_OK) return st;
  if ((st = make_map(&mz, workspace, static_cast<long long>(ws.nbuf) * B, p.c, f, rf::HALF)) != RA_OK) return st;
  if ((st = make_map(&mw2, w2, 1, p.h, f, rf::HALF)) != RA_OK) return st;
  const cudaError_t me = cudaMemsetAsync(p.ready, 0, ws.ctr_bytes, stream);
  if (me != cudaSuccess) return cuda_fail(static_cast<int>(me), "cudaMemsetAsync(ffn counters)");
  constexpr int smem = rf::Layout::ALLOC;
  if (!di->ffn_attr) {
    const cudaError_t e = cudaFuncSetAttribute(rf::ffn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return cuda_fail(static_cast<int>(e), "cudaFuncSetAttribute(ffn smem)");
    di->ffn_attr = true;
  }
  // CTA pairs, one CTA per SM at most, all resident; pairs take tiles in order from the launch's
  // counter, and a tile waits only on tiles before it
  const int pairs_max = di->sm_count / 2;
  const int pairs = p.n_items < pairs_max ? p.n_items : pairs_max;
  if (pairs < 1) return RA_ERR_DEVICE;
  rf::ffn_kernel<<<2 * pairs, rf::NUM_THREADS, smem, stream>>>(mx, mw1, mz, mw2, p);
  return launch_status();
}

}  // namespace

extern "C" {

size_t ring_attn_ffn_workspace_size(int B, int S, int D, int f) {
  if (B <= 0 || S <= 0 || D <= 0 || D > S || S % D != 0 || f <= 0) return 0;
  return ffn_workspace(B, S, D, f).total;
}

int ring_attn_ffn_block(const void* o, int B, int H, int S, int Dh, int D, int r, const void* w1, const float* b1,
                        const void* w2, const float* b2, int f, void* y, void* workspace, size_t workspace_bytes,
                        ra_stream stream) {
  int st = ffn_check(o, B, H, S, Dh, D, w1, b1, w2, b2, f, y, workspace, workspace_bytes);
  if (st != RA_OK) return st;
  if (r < 0 || r >= D) return RA_ERR_ARG;
  return ffn_run(o, B, H, S, Dh, D, r, 1, w1, b1, w2, b2, f, y, workspace, static_cast<cudaStream_t>(stream));
}

int ring_attn_ffn_fwd(const void* o, int B, int H, int S, int Dh, int D, const void* w1, const float* b1,
                      const void* w2, const float* b2, int f, void* y, void* workspace, size_t workspace_bytes,
                      ra_stream stream) {
  int st = ffn_check(o, B, H, S, Dh, D, w1, b1, w2, b2, f, y, workspace, workspace_bytes);
  if (st != RA_OK) return st;
  return ffn_run(o, B, H, S, Dh, D, 0, D, w1, b1, w2, b2, f, y, workspace, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
