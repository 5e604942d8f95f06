// C ABI of libringattn.so: argument validation, TMA descriptor construction and kernel
// launches on the caller's stream.  See include/ring_attn.h for the contract of every
// entry point.  No device memory is allocated here and nothing synchronises except
// ring_attn_device_status.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <climits>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "ring_attn.h"
#include "fwd_sm100.cuh"
#include "fwd_f32.cuh"
#include "merge.cuh"
#include "bwd_sm100.cuh"
#include "ffn_sm100.cuh"

namespace {

// Last failing CUDA call of this host thread (diagnostics for RA_ERR_CUDA).
thread_local int g_last_cuda_code = 0;
thread_local const char* g_last_cuda_site = "";

int cuda_fail(int code, const char* site) {
  g_last_cuda_code = code;
  g_last_cuda_site = site;
  return RA_ERR_CUDA;
}

constexpr int RA_VERSION = 100;

// Kernels this library has launched (all threads, all devices) since load.
std::atomic<unsigned long long> g_launches{0};
constexpr int MAX_DEVICES = 64;

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

struct DevInfo {
  int sm_count = 0;
  std::atomic<unsigned> next_work_slot{0};   // round robin over the kernels' work counters
  bool ok = false;          // compute capability 10.0
  // shared-memory attributes already set: [HD 128, HD 64] x [whole ring, split]; read and
  // written by any host thread, hence atomic (setting an attribute twice is harmless)
  std::atomic<bool> fwd_attr[4] = {false, false, false, false};
  std::atomic<bool> bwd_attr[2] = {false, false};   // [HD 128, HD 64]
  std::atomic<bool> ffn_attr{false};
};

std::mutex g_dev_mu;
DevInfo g_dev[MAX_DEVICES];
bool g_dev_init[MAX_DEVICES] = {};

// Current device's info (cached); nullptr on a CUDA failure.
DevInfo* dev_info(int* status) {
  int dev = 0;
  const cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) {
    *status = cuda_fail(static_cast<int>(e), "cudaGetDevice");
    return nullptr;
  }
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if (!g_dev_init[dev]) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      *status = RA_ERR_CUDA;
      return nullptr;
    }
    g_dev[dev].sm_count = sms;
    g_dev[dev].ok = (major == 10 && minor == 0);
    g_dev_init[dev] = true;
  }
  if (!g_dev[dev].ok) {
    *status = RA_ERR_DEVICE;
    return nullptr;
  }
  *status = RA_OK;
  return &g_dev[dev];
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// 3-D tensor map over a [BH][S][Dh] tensor (bf16, or fp32 when `f32`): box = 128 bytes of
// columns x `box_rows` rows x 1 head, 128-byte swizzle, zero fill outside [0, S) so tiles
// never read the next head (and stores/reductions there are dropped).
int make_map(CUtensorMap* map, const void* base, long long BH, int S, int Dh, int box_rows, bool f32 = false) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return cuda_fail(-1, "cudaGetDriverEntryPoint(cuTensorMapEncodeTiled)");
  const cuuint64_t esz = f32 ? 4 : 2;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(Dh), static_cast<cuuint64_t>(S), static_cast<cuuint64_t>(BH)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(Dh) * esz, static_cast<cuuint64_t>(S) * Dh * esz};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(128 / esz), static_cast<cuuint32_t>(box_rows), 1u};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  const CUresult r = enc(map, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                         const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? RA_OK : cuda_fail(static_cast<int>(r), "cuTensorMapEncodeTiled");
}

// Common shape checks.  Sizes are bounded so that every element index fits in int64 and
// every per-head row index fits in int.
int check_shape(int B, int H, int S, int Dh, int D) {
  if (B <= 0 || H <= 0 || S <= 0 || Dh <= 0 || D <= 0) return RA_ERR_ARG;
  if (D > S || S % D != 0) return RA_ERR_SHAPE;
  const long long BH = static_cast<long long>(B) * H;
  if (BH > INT_MAX / 2) return RA_ERR_SHAPE;
  if (static_cast<double>(BH) * S * Dh > 9.0e18 / 4) return RA_ERR_SHAPE;
  return RA_OK;
}

// Heads whose per-head streamed operands (`bytes_per_head`) fit together in `mib` MiB of L2.
#ifndef RA_L2_GROUP_MIB
#define RA_L2_GROUP_MIB 48          // backward: Q + dO of the heads in flight
#endif
#ifndef RA_FWD_L2_GROUP_MIB
#define RA_FWD_L2_GROUP_MIB 48      // forward: K + V of the heads in flight (0: all heads) ...
#endif
#ifndef RA_FWD_L2_GROUP_ABOVE_MIB
#define RA_FWD_L2_GROUP_ABOVE_MIB 256   // ... once K + V of all heads exceed this (about 2x L2)
#endif
int heads_per_l2_group(long long BH, long long bytes_per_head, long long mib = RA_L2_GROUP_MIB) {
  const long long g = (mib << 20) / (bytes_per_head > 0 ? bytes_per_head : 1);
  return static_cast<int>(g < 1 ? 1 : (g > BH ? BH : g));
}

int launch_status() {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? RA_OK : cuda_fail(static_cast<int>(e), "kernel launch");
}

// o_part given: each query pair's visit order is cut into n_parts pieces (n_parts >= 1),
// written as fp32 partials to o_part / lse_part ([n_parts][B*H][S][HD], [n_parts][B*H][S])
// for the merge; o and lse are then not written.
template <int HD>
int fwd_bf16(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int S, int D, int causal,
             float scale, cudaStream_t stream, int n_parts = 1, float* o_part = nullptr, float* lse_part = nullptr) {
  using namespace ra::fwd;
  int st = RA_OK;
  DevInfo* di = dev_info(&st);
  if (!di) return st;
  const long long BH = static_cast<long long>(B) * H;
  CUtensorMap mq, mk, mv;
  if ((st = make_map(&mq, q, BH, S, HD, BM)) != RA_OK) return st;
  if ((st = make_map(&mk, k, BH, S, HD, BN)) != RA_OK) return st;
  if ((st = make_map(&mv, v, BH, S, HD, BN)) != RA_OK) return st;
  Params p;
  p.BH = static_cast<int>(BH);
  p.S = S;
  p.D = D;
  p.causal = causal ? 1 : 0;
  p.n_pairs = (S + ROWS - 1) / ROWS;
  p.n_parts = n_parts;
  const long long items = BH * p.n_pairs * n_parts;
  if (items > INT_MAX) return RA_ERR_SHAPE;
  p.n_items = static_cast<int>(items);
  // Heads grouped so the K and V of the heads in flight fit in ~48 MiB of L2, once all heads'
  // K and V are well beyond L2.  Measured on B200 (0.5 s regions, clocks under the power cap):
  // S = 32K, 32 heads 1012 -> 1054 TFLOP/s and S = 128K, 8 heads 1083 -> 1095 (the DRAM traffic
  // falls and the SM clock rises ~100 MHz); at S = 16K, 16 heads (128 MiB of K and V) all heads
  // interleaved stays best (1012 against 962).
  const long long kv_head = 4ll * S * HD;   // K + V bytes of one head
  p.hgroup = (RA_FWD_L2_GROUP_MIB > 0 && BH * kv_head > (static_cast<long long>(RA_FWD_L2_GROUP_ABOVE_MIB) << 20))
                 ? heads_per_l2_group(BH, kv_head, RA_FWD_L2_GROUP_MIB)
                 : static_cast<int>(BH);
  p.work_slot = static_cast<int>(di->next_work_slot.fetch_add(1) % ra::WORK_SLOTS);
  p.scale_log2 = scale * 1.4426950408889634f;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.o_part = o_part;
  p.lse_part = lse_part;
  constexpr int smem = Layout<HD>::ALLOC;
  const bool split = o_part != nullptr;
  const int slot = (HD == 128 ? 0 : 1) + (split ? 2 : 0);
  auto kern = split ? fwd_kernel<HD, true> : fwd_kernel<HD, false>;
  if (!di->fwd_attr[slot]) {
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return cuda_fail(static_cast<int>(e), "cudaFuncSetAttribute(fwd smem)");
    di->fwd_attr[slot] = true;
  }
  const int grid = p.n_items < di->sm_count ? p.n_items : di->sm_count;
  kern<<<grid, NUM_THREADS, smem, stream>>>(mq, mk, mv, p);
  return launch_status();
}

int fwd_f32(const float* q, const float* k, const float* v, float* o, float* lse, int B, int H, int S, int Dh, int D,
            int causal, float scale, cudaStream_t stream) {
  using namespace ra::f32;
  const long long rows = static_cast<long long>(B) * H * S;
  const long long blocks = (rows + WARPS - 1) / WARPS;
  if (blocks > INT_MAX) return RA_ERR_SHAPE;
  const int vpl = (Dh + 31) / 32;
#define RA_F32_CASE(N)                                                                                         \
  case N:                                                                                                      \
    fwd_f32_kernel<N><<<static_cast<int>(blocks), WARPS * 32, 0, stream>>>(q, k, v, o, lse, rows, S, Dh, D,  \
                                                                           causal, scale);                   \
    break;
  switch (vpl) {
    RA_F32_CASE(1) RA_F32_CASE(2) RA_F32_CASE(3) RA_F32_CASE(4) RA_F32_CASE(5) RA_F32_CASE(6) RA_F32_CASE(7)
    RA_F32_CASE(8)
    default:
      return RA_ERR_SHAPE;
  }
#undef RA_F32_CASE
  return launch_status();
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct BwdWorkspace {
  size_t dq_bytes, row_bytes, total;
};

BwdWorkspace bwd_workspace(long long BH, int S, int Dh) {
  const long long S_pad = (static_cast<long long>(S) + 127) / 128 * 128;
  BwdWorkspace w;
  w.dq_bytes = align256(static_cast<size_t>(BH) * S * Dh * 4);
  w.row_bytes = align256(static_cast<size_t>(BH) * S_pad * 4);
  w.total = w.dq_bytes + 2 * w.row_bytes;
  return w;
}

// dq32 given: dQ, dK, dV are added to the fp32 dq32, dk32, dv32 instead of written to the
// bf16 dq, dk, dv.
template <int HD>
int bwd_bf16(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO, void* dq,
             void* dk, void* dv, int B, int H, int S, int D, int causal, float scale, void* workspace,
             cudaStream_t stream, float* dq32 = nullptr, float* dk32 = nullptr, float* dv32 = nullptr) {
  namespace rb = ra::bwd;
  int st = RA_OK;
  DevInfo* di = dev_info(&st);
  if (!di) return st;
  const long long BH = static_cast<long long>(B) * H;
  const BwdWorkspace ws = bwd_workspace(BH, S, HD);
  const int S_pad = (S + 127) / 128 * 128;
  float* dq_acc = static_cast<float*>(workspace);
  float* delta = reinterpret_cast<float*>(static_cast<char*>(workspace) + ws.dq_bytes);
  float* lse2 = reinterpret_cast<float*>(static_cast<char*>(workspace) + ws.dq_bytes + ws.row_bytes);

  // 1. Delta, lse * log2(e), cleared dQ accumulator
  const long long prow = BH * S_pad;
  const long long pre_blocks = (prow + rb::PRE_WARPS - 1) / rb::PRE_WARPS;
  if (pre_blocks > INT_MAX) return RA_ERR_SHAPE;
  rb::bwd_pre_kernel<HD><<<static_cast<int>(pre_blocks), rb::PRE_WARPS * 32, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dO), lse, delta, lse2, dq_acc,
      static_cast<int>(BH), S, S_pad);
  if ((st = launch_status()) != RA_OK) return st;

  // 2. key/value-stationary main kernel
  CUtensorMap mq, mk, mv, mdo;
  if ((st = make_map(&mq, q, BH, S, HD, rb::BQ)) != RA_OK) return st;
  if ((st = make_map(&mk, k, BH, S, HD, rb::BM)) != RA_OK) return st;
  if ((st = make_map(&mv, v, BH, S, HD, rb::BM)) != RA_OK) return st;
  if ((st = make_map(&mdo, dO, BH, S, HD, rb::BQ)) != RA_OK) return st;
  CUtensorMap mdq;   // fp32 accumulator, 32-column boxes for the reduce-adds
  if ((st = make_map(&mdq, dq_acc, BH, S, HD, rb::BQ, true)) != RA_OK) return st;
  rb::Params p;
  p.BH = static_cast<int>(BH);
  p.S = S;
  p.S_pad = S_pad;
  p.D = D;
  p.causal = causal ? 1 : 0;
  p.n_kt = (S + rb::BM - 1) / rb::BM;
  const long long items = BH * p.n_kt;
  if (items > INT_MAX) return RA_ERR_SHAPE;
  p.n_items = static_cast<int>(items);
  p.hgroup = heads_per_l2_group(BH, 4ll * S * HD);   // Q + dO bytes of one head
  p.work_slot = static_cast<int>(di->next_work_slot.fetch_add(1) % ra::WORK_SLOTS);
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.lse2 = lse2;
  p.delta = delta;
  p.dq_acc = dq_acc;
  p.dk = static_cast<__nv_bfloat16*>(dk);
  p.dv = static_cast<__nv_bfloat16*>(dv);
  p.dk32 = dq32 ? dk32 : nullptr;
  p.dv32 = dq32 ? dv32 : nullptr;
  constexpr int smem = rb::Layout<HD>::BYTES;
  constexpr int aslot = HD == 128 ? 0 : 1;
  if (!di->bwd_attr[aslot]) {
    const cudaError_t e = cudaFuncSetAttribute(rb::bwd_kernel<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return cuda_fail(static_cast<int>(e), "cudaFuncSetAttribute(bwd smem)");
    di->bwd_attr[aslot] = true;
  }
  const int grid = p.n_items < di->sm_count ? p.n_items : di->sm_count;
  rb::bwd_kernel<HD><<<grid, rb::NUM_THREADS, smem, stream>>>(mq, mk, mv, mdo, mdq, p);
  if ((st = launch_status()) != RA_OK) return st;

  // 3. dQ = scale * accumulator -> bf16 (or added to dq32)
  if (dq32) {
    const long long n4 = BH * S * HD / 4;
    const long long ablocks = (n4 + 255) / 256;
    if (ablocks > INT_MAX) return RA_ERR_SHAPE;
    rb::bwd_accum_dq_kernel<<<static_cast<int>(ablocks), 256, 0, stream>>>(dq_acc, dq32, n4, scale);
    return launch_status();
  }
  const long long n8 = BH * S * HD / 8;
  const long long cblocks = (n8 + 255) / 256;
  if (cblocks > INT_MAX) return RA_ERR_SHAPE;
  rb::bwd_convert_kernel<<<static_cast<int>(cblocks), 256, 0, stream>>>(dq_acc, static_cast<__nv_bfloat16*>(dq), n8,
                                                                       scale);
  return launch_status();
}

// One thread waits, through the kernels' own bounded wait, on an mbarrier nothing arrives on.
__global__ void wait_selftest_kernel(unsigned long long timeout_ns) {
  __shared__ __align__(8) unsigned long long bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    ra::mbar_init(ra::smem_u32(&bar), 1);
    abort_flag = 0;
    ra::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) ra::mbar_wait(ra::smem_u32(&bar), 0, &abort_flag, timeout_ns);
}

__global__ void exp2_check_kernel(const float* __restrict__ x, float* __restrict__ y_fma, float* __restrict__ y_mufu,
                                  long long n) {
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < n) {
    y_fma[i] = ra::exp2_fma(x[i]);
    y_mufu[i] = ra::ex2_approx(x[i]);
  }
}

}  // namespace

extern "C" {

int ring_attn_wait_selftest(long long timeout_ns, ra_stream stream) {
  if (timeout_ns <= 0 || timeout_ns > 10000000000ll) return RA_ERR_ARG;
  int st = RA_OK;
  if (!dev_info(&st)) return st;
  wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<unsigned long long>(timeout_ns));
  return launch_status();
}

int ring_attn_exp2_check(const float* x, float* y_fma, float* y_mufu, long long n, ra_stream stream) {
  if (!x || !y_fma || !y_mufu || n <= 0) return RA_ERR_ARG;
  int st = RA_OK;
  if (!dev_info(&st)) return st;
  const long long blocks = (n + 255) / 256;
  if (blocks > INT_MAX) return RA_ERR_SHAPE;
  exp2_check_kernel<<<static_cast<int>(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y_fma, y_mufu, n);
  return launch_status();
}

int ring_attn_version(void) { return RA_VERSION; }

int ring_attn_last_cuda_error(const char** site) {
  if (site) *site = g_last_cuda_site;
  return g_last_cuda_code;
}

const char* ring_attn_strerror(int code) {
  switch (code) {
    case RA_OK: return "ok";
    case RA_ERR_ARG: return "invalid argument (null pointer, non-positive size or unknown dtype)";
    case RA_ERR_SHAPE: return "unsupported shape (S % D != 0, D > S, unsupported head dim or size overflow)";
    case RA_ERR_ALIGN: return "pointer not 16-byte aligned";
    case RA_ERR_WORKSPACE: return "workspace missing or too small";
    case RA_ERR_CUDA: return "CUDA runtime/driver call failed";
    case RA_ERR_TIMEOUT: return "a kernel gave up on a bounded internal wait";
    case RA_ERR_DEVICE: return "current device is not an sm_100 (B200-class) GPU";
    default: return "unknown status code";
  }
}

int ring_attn_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int S, int Dh,
                     int D, int causal, ra_dtype dtype, float scale, ra_stream stream) {
  if (!q || !k || !v || !o || !lse) return RA_ERR_ARG;
  if (dtype != RA_BF16 && dtype != RA_F32) return RA_ERR_ARG;
  int st = check_shape(B, H, S, Dh, D);
  if (st != RA_OK) return st;
  const float sc = (scale > 0.f && std::isfinite(scale)) ? scale : 1.0f / std::sqrt(static_cast<float>(Dh));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dtype == RA_F32) {
    if (Dh > 256) return RA_ERR_SHAPE;
    int dst = RA_OK;
    if (!dev_info(&dst)) return dst;
    return fwd_f32(static_cast<const float*>(q), static_cast<const float*>(k), static_cast<const float*>(v),
                   static_cast<float*>(o), lse, B, H, S, Dh, D, causal, sc, s);
  }
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return RA_ERR_ALIGN;
  if (Dh == 128) return fwd_bf16<128>(q, k, v, o, lse, B, H, S, D, causal, sc, s);
  if (Dh == 64) return fwd_bf16<64>(q, k, v, o, lse, B, H, S, D, causal, sc, s);
  return RA_ERR_SHAPE;
}

int ring_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int S, int Dh, int D,
                  int causal, ra_stream stream) {
  return ring_attn_fwd_ex(q, k, v, o, lse, B, H, S, Dh, D, causal, RA_BF16, 0.f, stream);
}

size_t ring_attn_fwd_split_workspace_size(int B, int H, int S, int Dh, int n_parts) {
  if (B <= 0 || H <= 0 || S <= 0 || Dh <= 0 || n_parts <= 0) return 0;
  const size_t rows = static_cast<size_t>(B) * H * S;
  // fp32 partial O, then the partial lse, each part's block 256-B aligned
  const size_t o_bytes = (rows * Dh * 4 + 255) / 256 * 256;
  const size_t l_bytes = (rows * 4 + 255) / 256 * 256;
  return static_cast<size_t>(n_parts) * (o_bytes + l_bytes);
}

int ring_attn_fwd_split(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int S, int Dh,
                        int D, int causal, int n_parts, void* workspace, size_t workspace_bytes, ra_stream stream) {
  if (!q || !k || !v || !o || !lse) return RA_ERR_ARG;
  if (n_parts <= 0 || n_parts > RA_MAX_FWD_PARTS) return RA_ERR_ARG;
  int st = check_shape(B, H, S, Dh, D);
  if (st != RA_OK) return st;
  if (Dh != 128 && Dh != 64) return RA_ERR_SHAPE;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return RA_ERR_ALIGN;
  const float sc = 1.f / std::sqrt(static_cast<float>(Dh));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (n_parts == 1) return Dh == 128 ? fwd_bf16<128>(q, k, v, o, lse, B, H, S, D, causal, sc, s)
                                     : fwd_bf16<64>(q, k, v, o, lse, B, H, S, D, causal, sc, s);
  const size_t need = ring_attn_fwd_split_workspace_size(B, H, S, Dh, n_parts);
  if (!workspace || workspace_bytes < need) return RA_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) % 256 != 0) return RA_ERR_ALIGN;
  const size_t rows = static_cast<size_t>(B) * H * S;
  const size_t o_bytes = (rows * Dh * 4 + 255) / 256 * 256;
  float* o_part = static_cast<float*>(workspace);
  float* lse_part = reinterpret_cast<float*>(static_cast<char*>(workspace) + static_cast<size_t>(n_parts) * o_bytes);
  // the merge reads part p at o_part + p * rows * Dh: keep the parts densely packed
  if (o_bytes != rows * Dh * 4) return RA_ERR_SHAPE;
  st = Dh == 128 ? fwd_bf16<128>(q, k, v, o, lse, B, H, S, D, causal, sc, s, n_parts, o_part, lse_part)
                 : fwd_bf16<64>(q, k, v, o, lse, B, H, S, D, causal, sc, s, n_parts, o_part, lse_part);
  if (st != RA_OK) return st;
  return ring_attn_merge(o_part, lse_part, n_parts, o, lse, B, H, S, Dh, stream);
}

int ring_attn_fwd_partial(const void* q, const void* k, const void* v, float* o_part, float* lse_part, int B, int H,
                          int S, int Dh, int D, int causal, ra_stream stream) {
  if (!q || !k || !v || !o_part || !lse_part) return RA_ERR_ARG;
  int st = check_shape(B, H, S, Dh, D);
  if (st != RA_OK) return st;
  if (Dh != 128 && Dh != 64) return RA_ERR_SHAPE;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o_part)) return RA_ERR_ALIGN;
  const float sc = 1.f / std::sqrt(static_cast<float>(Dh));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // one piece: the split kernel's fp32 epilogue over the whole visit order
  return Dh == 128 ? fwd_bf16<128>(q, k, v, nullptr, nullptr, B, H, S, D, causal, sc, s, 1, o_part, lse_part)
                   : fwd_bf16<64>(q, k, v, nullptr, nullptr, B, H, S, D, causal, sc, s, 1, o_part, lse_part);
}

int ring_attn_merge_ex(const float* o_parts, const float* lse_parts, int P, void* o, float* lse, int B, int H, int S,
                       int Dh, ra_dtype out_dtype, ra_stream stream) {
  if (!o_parts || !lse_parts || !o || !lse) return RA_ERR_ARG;
  if (P <= 0 || B <= 0 || H <= 0 || S <= 0 || Dh <= 0) return RA_ERR_ARG;
  if (out_dtype != RA_BF16 && out_dtype != RA_F32) return RA_ERR_ARG;
  if (Dh % 4 != 0 || Dh > 256) return RA_ERR_SHAPE;
  if (!aligned16(o_parts) || !aligned16(o)) return RA_ERR_ALIGN;
  const long long rows = static_cast<long long>(B) * H * S;
  if (static_cast<double>(rows) * P * Dh > 9.0e18 / 4) return RA_ERR_SHAPE;
  int st = RA_OK;
  DevInfo* di = dev_info(&st);
  if (!di) return st;
  // grid capped at BLOCKS_PER_SM blocks per SM; the kernel strides over the rows
  long long blocks = (rows + ra::merge::WARPS - 1) / ra::merge::WARPS;
  const long long cap = static_cast<long long>(di->sm_count) * ra::merge::BLOCKS_PER_SM;
  if (blocks > cap) blocks = cap;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (out_dtype == RA_BF16)
    ra::merge::merge_kernel<__nv_bfloat16><<<static_cast<int>(blocks), ra::merge::WARPS * 32, 0, s>>>(
        o_parts, lse_parts, P, static_cast<__nv_bfloat16*>(o), lse, rows, Dh);
  else
    ra::merge::merge_kernel<float><<<static_cast<int>(blocks), ra::merge::WARPS * 32, 0, s>>>(
        o_parts, lse_parts, P, static_cast<float*>(o), lse, rows, Dh);
  return launch_status();
}

int ring_attn_merge(const float* o_parts, const float* lse_parts, int P, void* o, float* lse, int B, int H, int S,
                    int Dh, ra_stream stream) {
  return ring_attn_merge_ex(o_parts, lse_parts, P, o, lse, B, H, S, Dh, RA_BF16, stream);
}

int ring_attn_ring_order(int D, int r, int causal, int* blocks, int max_blocks) {
  if (D <= 0 || r < 0 || r >= D || !blocks) return -RA_ERR_ARG;
  int n = 0;
  for (int t = 0; t < D; ++t) {
    const int j = ((r - t) % D + D) % D;
    if (causal && j > r) continue;
    if (n >= max_blocks) return -RA_ERR_ARG;
    blocks[n++] = j;
  }
  return n;
}

int ring_attn_visit_tiles(int S, int D, int causal, int q0, int tile_rows, int* tiles, int max_tiles) {
  if (S <= 0 || D <= 0 || D > S || S % D != 0 || q0 < 0 || q0 >= S || tile_rows <= 0 || !tiles)
    return -RA_ERR_ARG;
  ra::RingTiles it;
  it.init(S, D, causal, q0, tile_rows, ra::fwd::BN);
  int n = 0;
  for (int kt = it.next(); kt >= 0; kt = it.next()) {
    if (n >= max_tiles) return -RA_ERR_ARG;
    tiles[n++] = kt;
  }
  return n;
}

int ring_attn_device_status(ra_stream stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return RA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, ra::g_status, sizeof(int)) != cudaSuccess) return RA_ERR_CUDA;
  if (v != 0) {
    const int z = 0;
    if (cudaMemcpyToSymbol(ra::g_status, &z, sizeof(int)) != cudaSuccess) return RA_ERR_CUDA;
  }
  return v;
}

}  // extern "C"


extern "C" {

size_t ring_attn_bwd_workspace_size(int B, int H, int S, int Dh) {
  if (B <= 0 || H <= 0 || S <= 0 || Dh <= 0) return 0;
  return bwd_workspace(static_cast<long long>(B) * H, S, Dh).total;
}

int ring_attn_bwd_ex(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
                     void* dq, void* dk, void* dv, int B, int H, int S, int Dh, int D, int causal, float scale,
                     void* workspace, size_t workspace_bytes, ra_stream stream) {
  if (!q || !k || !v || !o || !lse || !dO || !dq || !dk || !dv) return RA_ERR_ARG;
  int st = check_shape(B, H, S, Dh, D);
  if (st != RA_OK) return st;
  if (Dh != 128 && Dh != 64) return RA_ERR_SHAPE;
  for (const void* ptr : {q, k, v, o, dO, static_cast<const void*>(dq), static_cast<const void*>(dk),
                          static_cast<const void*>(dv)})
    if (!aligned16(ptr)) return RA_ERR_ALIGN;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 ||
      workspace_bytes < ring_attn_bwd_workspace_size(B, H, S, Dh))
    return RA_ERR_WORKSPACE;
  const float sc = (scale > 0.f && std::isfinite(scale)) ? scale : 1.0f / std::sqrt(static_cast<float>(Dh));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return Dh == 128 ? bwd_bf16<128>(q, k, v, o, lse, dO, dq, dk, dv, B, H, S, D, causal, sc, workspace, s)
                   : bwd_bf16<64>(q, k, v, o, lse, dO, dq, dk, dv, B, H, S, D, causal, sc, workspace, s);
}

int ring_attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
                  void* dq, void* dk, void* dv, int B, int H, int S, int Dh, int D, int causal, void* workspace,
                  size_t workspace_bytes, ra_stream stream) {
  return ring_attn_bwd_ex(q, k, v, o, lse, dO, dq, dk, dv, B, H, S, Dh, D, causal, 0.f, workspace,
                          workspace_bytes, stream);
}

int ring_attn_bwd_accumulate(const void* q, const void* k, const void* v, const void* o, const float* lse,
                             const void* dO, float* dq32, float* dk32, float* dv32, int B, int H, int S, int Dh, int D,
                             int causal, void* workspace, size_t workspace_bytes, ra_stream stream) {
  if (!q || !k || !v || !o || !lse || !dO || !dq32 || !dk32 || !dv32) return RA_ERR_ARG;
  int st = check_shape(B, H, S, Dh, D);
  if (st != RA_OK) return st;
  if (Dh != 128 && Dh != 64) return RA_ERR_SHAPE;
  for (const void* ptr : {q, k, v, o, dO, static_cast<const void*>(dq32), static_cast<const void*>(dk32),
                          static_cast<const void*>(dv32)})
    if (!aligned16(ptr)) return RA_ERR_ALIGN;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 ||
      workspace_bytes < ring_attn_bwd_workspace_size(B, H, S, Dh))
    return RA_ERR_WORKSPACE;
  const float sc = 1.0f / std::sqrt(static_cast<float>(Dh));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return Dh == 128 ? bwd_bf16<128>(q, k, v, o, lse, dO, nullptr, nullptr, nullptr, B, H, S, D, causal, sc, workspace,
                                   s, dq32, dk32, dv32)
                   : bwd_bf16<64>(q, k, v, o, lse, dO, nullptr, nullptr, nullptr, B, H, S, D, causal, sc, workspace,
                                  s, dq32, dk32, dv32);
}

int ring_attn_bwd_visit_tiles(int S, int D, int causal, int k0, int tile_rows, int* tiles, int max_tiles) {
  if (S <= 0 || D <= 0 || D > S || S % D != 0 || k0 < 0 || k0 >= S || tile_rows <= 0 || !tiles)
    return -RA_ERR_ARG;
  ra::RingQTiles it;
  it.init(S, D, causal, k0, tile_rows);
  int n = 0;
  for (int qt = it.next(); qt >= 0; qt = it.next()) {
    if (n >= max_tiles) return -RA_ERR_ARG;
    tiles[n++] = qt;
  }
  return n;
}

unsigned long long ring_attn_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

}  // extern "C"

// --- backward without caller-provided workspace -------------------------------------------
// Scratch for ring_attn_bwd_noalloc: the fp32 dQ accumulator and the two per-row statistics
// live in this file-scope device array instead of a caller buffer.  Every device that loads
// the library holds RA_NOALLOC_SCRATCH_BYTES for it until the process exits.
namespace {

constexpr size_t RA_NOALLOC_SCRATCH_BYTES = 96ull << 20;   // 96 MiB per device
static __device__ __align__(256) unsigned char g_noalloc_scratch[RA_NOALLOC_SCRATCH_BYTES];

std::mutex g_scratch_mu;
void* g_scratch_ptr[MAX_DEVICES] = {};

// Device address of the scratch array on the current device, looked up once per device
// (host code may not use the array's name as a device pointer).
int scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) return cuda_fail(static_cast<int>(e), "cudaGetDevice");
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) return cuda_fail(static_cast<int>(e), "cudaGetSymbolAddress(noalloc scratch)");
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return RA_OK;
}

}  // namespace

extern "C" {

size_t ring_attn_bwd_noalloc_max_bytes(void) { return RA_NOALLOC_SCRATCH_BYTES; }

int ring_attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                          const void* dO, void* dq, void* dk, void* dv, int B, int H, int S, int Dh, int D,
                          int causal, ra_stream stream) {
  if (!q || !k || !v || !o || !lse || !dO || !dq || !dk || !dv) return RA_ERR_ARG;
  int st = check_shape(B, H, S, Dh, D);
  if (st != RA_OK) return st;
  if (Dh != 128 && Dh != 64) return RA_ERR_SHAPE;
  for (const void* ptr : {q, k, v, o, dO, static_cast<const void*>(dq), static_cast<const void*>(dk),
                          static_cast<const void*>(dv)})
    if (!aligned16(ptr)) return RA_ERR_ALIGN;
  if (ring_attn_bwd_workspace_size(B, H, S, Dh) > RA_NOALLOC_SCRATCH_BYTES) return RA_ERR_WORKSPACE;
  int dst = RA_OK;
  if (!dev_info(&dst)) return dst;
  void* scratch = nullptr;
  if ((st = scratch_address(&scratch)) != RA_OK) return st;
  const float sc = 1.0f / std::sqrt(static_cast<float>(Dh));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return Dh == 128 ? bwd_bf16<128>(q, k, v, o, lse, dO, dq, dk, dv, B, H, S, D, causal, sc, scratch, s)
                   : bwd_bf16<64>(q, k, v, o, lse, dO, dq, dk, dv, B, H, S, D, causal, sc, scratch, s);
}

}  // extern "C"

// The blockwise feedforward's host side (workspace, checks, launch, entry points).
#include "ffn_host.cuh"
