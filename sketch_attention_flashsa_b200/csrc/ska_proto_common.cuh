// Helpers shared by the prototype-wise forward kernels: the walk over the concatenated
// (user, head) tile stream and the bounded mbarrier wait.
#pragma once

#include "ska_internal.h"
#include "ska_ptx.cuh"

namespace ska {

// Position in the concatenated tile stream: segment (b, h), tile j of user b.
struct TilePos {
  int b, h, j, nb;  // nb = tiles of user b
  int g;            // global tile index
};

__device__ __forceinline__ int user_used(const ProtoFwdParams& p, int b) {
  int len = p.cu_seqlens[b + 1] - p.cu_seqlens[b];
  if (p.seqused) len = min(len, p.seqused[b]);
  return max(len, 0);
}

__device__ __forceinline__ void tile_seek(const ProtoFwdParams& p, int g, TilePos& t) {
  // largest b in [0, B) with H * prefix[b] <= g
  int lo = 0, hi = p.B - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (p.H * p.tile_prefix[mid] <= g) lo = mid; else hi = mid - 1;
  }
  t.b = lo;
  t.nb = p.tile_prefix[lo + 1] - p.tile_prefix[lo];
  int off = g - p.H * p.tile_prefix[lo];
  t.h = off / t.nb;
  t.j = off - t.h * t.nb;
  t.g = g;
}

__device__ __forceinline__ void tile_next(const ProtoFwdParams& p, TilePos& t) {
  t.g++;
  if (++t.j < t.nb) return;
  t.j = 0;
  if (++t.h < p.H) return;
  t.h = 0;
  do {
    t.b++;
    if (t.b >= p.B) return;
    t.nb = p.tile_prefix[t.b + 1] - p.tile_prefix[t.b];
  } while (t.nb == 0);
}

struct Waiter {
  int* abort_flag;  // the CTA's abort flag in shared memory
  int* status;
  uint64_t budget;
  // Bounded wait; on timeout records the error and raises the CTA's abort flag. Unless
  // `drain` is set, a raised abort flag ends the wait early; drains (waiting for this
  // thread's own copies and MMAs in flight before exit) only end on completion or budget.
  __device__ __forceinline__ bool operator()(uint64_t* bar, uint32_t parity, bool cluster_scope = false,
                                             bool drain = false) {
    volatile int* ab = abort_flag;
    bool ok = cluster_scope ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity);
    if (ok) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
      ok = cluster_scope ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity);
      if (ok) return true;
      if (!drain && *ab) return false;
      if (globaltimer_ns() - t0 > budget) {
        atomicCAS(status, 0, (int)SKA_ERR_DEVICE_TIMEOUT);
        *ab = 1;
        return false;
      }
    }
  }
};

}  // namespace ska
