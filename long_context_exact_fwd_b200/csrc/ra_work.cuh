// Dynamic work distribution for the persistent kernels.
//
// Work items are numbered longest first; CTAs take the next number from a global counter as
// they become free (greedy longest-processing-time scheduling), instead of a fixed
// round-robin share that leaves some SMs with far more causal work than others.
//
// Counters: g_work[slot] = {next item, CTAs finished}.  The host gives every launch its own
// slot (round robin over WORK_SLOTS per device), so launches that are in flight together on
// different streams never share one.  Each CTA bumps "finished" once, after its last fetch;
// the CTA that completes the count resets both words, leaving the slot at zero for the launch
// that reuses it WORK_SLOTS launches later.
//
// Inside a CTA one thread fetches and publishes item numbers through a two-entry ring in
// shared memory guarded by mbarriers; every other role pops the same sequence.
#pragma once
#include "ra_sm100.cuh"

namespace ra {

constexpr int WORK_SLOTS = 256;
__device__ unsigned int g_work[WORK_SLOTS][2];

__device__ __forceinline__ int work_fetch(int slot) { return static_cast<int>(atomicAdd(&g_work[slot][0], 1u)); }

// Called once per CTA by the fetching thread after its final fetch (also on abort paths).
__device__ __forceinline__ void work_done(int slot) {
  __threadfence();
  if (atomicAdd(&g_work[slot][1], 1u) == gridDim.x - 1) {
    atomicExch(&g_work[slot][0], 0u);
    atomicExch(&g_work[slot][1], 0u);
  }
}

// Shared-memory ring of item numbers.  full[i] completes when entry i is written (1 arrival);
// empty[i] completes when every consumer has read it (`consumers` arrivals).
struct ItemRing {
  uint32_t full;        // shared address of full[0]; full[1] is 8 bytes further
  uint32_t empty;       // shared address of empty[0]
  volatile int* slot;   // two entries
  int k = 0;
  uint32_t ph = 0;

  __device__ __forceinline__ void advance() {
    if (++k == 2) {
      k = 0;
      ph ^= 1u;
    }
  }

  // Producer: publish `item` (waits until the entry's previous value has been read).
  __device__ __forceinline__ bool push(int item, volatile int* abort_flag) {
    if (!mbar_wait(empty + 8u * k, ph ^ 1u, abort_flag)) return false;
    slot[k] = item;
    mbar_arrive(full + 8u * k);
    advance();
    return true;
  }

  // Single-thread consumer.
  __device__ __forceinline__ bool pop(int& item, volatile int* abort_flag) {
    if (!mbar_wait(full + 8u * k, ph, abort_flag)) return false;
    item = slot[k];
    mbar_arrive(empty + 8u * k);
    advance();
    return true;
  }

  // Warp consumer: all 32 lanes read, lane 0 arrives once for the warp.  The outcome is
  // uniform across the warp.
  __device__ __forceinline__ bool pop_warp(int& item, volatile int* abort_flag) {
    const bool ok = __all_sync(0xffffffffu, mbar_wait(full + 8u * k, ph, abort_flag));
    if (!ok) return false;
    item = slot[k];
    __syncwarp();
    if ((threadIdx.x & 31u) == 0u) mbar_arrive(empty + 8u * k);
    advance();
    return true;
  }
};

}  // namespace ra
