// Device-side sketch cache (SequenceO1 §4.1): the user-only sketch X~_u is cached, keyed by
// (user id, model version, history timestamp, sketch configuration), with TTL invalidation and
// capacity eviction, behind one get/put interface for training and serving.
//
// The cache is set-associative: S sets (a power of two) of W <= 32 ways. A key's set is SplitMix64
// (Steele, Lea and Flood 2014; z = x + 0x9E3779B97F4A7C15, then the xor-shift-multiply mix) applied
// in turn to the user id, version, configuration and timestamp, masked to S - 1.
//   get: a key hits when a way of its set holds it, stored at time t with now - t <= ttl. The
//        stored row is copied out; a miss gives a zero row.
//   put: keys are applied in batch order. A way holding the same key is overwritten; otherwise the
//        first empty or expired way is used, failing that the oldest (ties: the lowest way).
// One warp serves one key, one lane per way. A put batch runs in three steps:
//   1. every key counts itself into its set;
//   2. keys alone in their set decide in parallel, and the keys of shared sets are applied by one
//      warp in batch order, recording the last key written to each slot;
//   3. each key copies its row unless a later key of the batch took its slot.
// No step waits on another CTA.
#include <algorithm>
#include <climits>

#include "ska_internal.h"

namespace ska {

namespace {

constexpr int64_t kEmpty = LLONG_MIN;

struct CacheEntry {  // 32 bytes
  uint64_t user;
  uint32_t version;
  uint32_t config;
  int64_t timestamp;
  int64_t stamp;     // time of the put; kEmpty when the way holds nothing
};

struct CacheLayout {
  size_t entries, counts, owner, data, total;
};

__host__ __device__ inline CacheLayout cache_layout(const ska_cache_desc& d) {
  CacheLayout L;
  const size_t slots = size_t(d.num_sets) * d.ways;
  size_t off = 256;
  L.entries = off;
  off += slots * sizeof(CacheEntry);
  L.counts = off;
  off += ((size_t(d.num_sets) * 4 + 255) / 256) * 256;
  L.owner = off;
  off += ((slots * 4 + 255) / 256) * 256;
  L.data = off;
  off += slots * size_t(d.row_floats) * 4;
  L.total = off;
  return L;
}

__device__ __forceinline__ uint64_t splitmix64(uint64_t x) {
  uint64_t z = x + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__device__ __forceinline__ int cache_set(const ska_cache_key& k, int num_sets) {
  uint64_t h = splitmix64(k.user_id);
  h = splitmix64(h ^ k.model_version);
  h = splitmix64(h ^ k.sketch_config);
  h = splitmix64(h ^ static_cast<uint64_t>(k.history_timestamp));
  return static_cast<int>(h & static_cast<uint64_t>(num_sets - 1));
}

__device__ __forceinline__ bool same_key(const CacheEntry& e, const ska_cache_key& k) {
  return e.user == k.user_id && e.version == k.model_version && e.config == k.sketch_config &&
         e.timestamp == k.history_timestamp;
}

__device__ __forceinline__ bool live(const CacheEntry& e, int64_t now, int64_t ttl) {
  return e.stamp != kEmpty && now - e.stamp <= ttl;
}

// The way a put of key k at `now` writes to, decided by the warp (lane w reads way w).
__device__ __forceinline__ int choose_way(const CacheEntry* set_entries, int W, const ska_cache_key& k, int64_t now,
                                          int64_t ttl) {
  const int lane = threadIdx.x & 31;
  CacheEntry e{};
  e.stamp = kEmpty;
  if (lane < W) e = set_entries[lane];
  const uint32_t mine = __ballot_sync(0xffffffffu, lane < W && e.stamp != kEmpty && same_key(e, k));
  if (mine) return __ffs(mine) - 1;
  const uint32_t free_ways = __ballot_sync(0xffffffffu, lane < W && !live(e, now, ttl));
  if (free_ways) return __ffs(free_ways) - 1;
  // the oldest way, the lowest index among equal times
  int64_t best = (lane < W) ? e.stamp : LLONG_MAX;
  int bw = lane;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const int64_t ob = __shfl_xor_sync(0xffffffffu, best, o);
    const int ow = __shfl_xor_sync(0xffffffffu, bw, o);
    if (ob < best || (ob == best && ow < bw)) {
      best = ob;
      bw = ow;
    }
  }
  return bw;
}

__global__ void cache_init_kernel(CacheEntry* entries, int64_t slots) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < slots;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    CacheEntry e{};
    e.stamp = kEmpty;
    entries[i] = e;
  }
}

__global__ void cache_count_kernel(const ska_cache_key* keys, int n, int num_sets, int32_t* counts) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x)
    atomicAdd(&counts[cache_set(keys[i], num_sets)], 1);
}

// Keys alone in their set: one warp each, in parallel.
__global__ void cache_put_unique_kernel(ska_cache_desc d, CacheEntry* entries, const int32_t* counts,
                                        const ska_cache_key* keys, int n, int64_t now, int32_t* slots) {
  const int warps = (gridDim.x * blockDim.x) >> 5;
  for (int i = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; i < n; i += warps) {
    const ska_cache_key k = keys[i];
    const int s = cache_set(k, d.num_sets);
    if (counts[s] != 1) continue;  // warp-uniform
    CacheEntry* se = entries + static_cast<int64_t>(s) * d.ways;
    const int w = choose_way(se, d.ways, k, now, d.ttl);
    if ((threadIdx.x & 31) == 0) {
      CacheEntry e;
      e.user = k.user_id;
      e.version = k.model_version;
      e.config = k.sketch_config;
      e.timestamp = k.history_timestamp;
      e.stamp = now;
      se[w] = e;
      slots[i] = s * d.ways + w;
    }
  }
}

// Keys whose set holds other keys of the batch: one warp applies them in batch order and records
// the last key written to each slot. The warp scans 32 keys at a time and applies the ones in shared
// sets one after another.
__global__ void cache_put_shared_kernel(ska_cache_desc d, CacheEntry* entries, const int32_t* counts, int32_t* owner,
                                        const ska_cache_key* keys, int n, int64_t now, int32_t* slots) {
  if (blockIdx.x != 0 || threadIdx.x >= 32) return;
  const int lane = threadIdx.x;
  for (int base = 0; base < n; base += 32) {
    const int i = base + lane;
    ska_cache_key k{};
    int s = 0;
    bool shared = false;
    if (i < n) {
      k = keys[i];
      s = cache_set(k, d.num_sets);
      shared = counts[s] != 1;
    }
    uint32_t m = __ballot_sync(0xffffffffu, shared);
    while (m) {
      const int src = __ffs(m) - 1;
      m &= m - 1;
      ska_cache_key kk;
      kk.user_id = __shfl_sync(0xffffffffu, k.user_id, src);
      kk.model_version = __shfl_sync(0xffffffffu, k.model_version, src);
      kk.sketch_config = __shfl_sync(0xffffffffu, k.sketch_config, src);
      kk.history_timestamp = __shfl_sync(0xffffffffu, k.history_timestamp, src);
      const int ss = __shfl_sync(0xffffffffu, s, src);
      CacheEntry* se = entries + static_cast<int64_t>(ss) * d.ways;
      const int w = choose_way(se, d.ways, kk, now, d.ttl);
      if (lane == 0) {
        CacheEntry e;
        e.user = kk.user_id;
        e.version = kk.model_version;
        e.config = kk.sketch_config;
        e.timestamp = kk.history_timestamp;
        e.stamp = now;
        se[w] = e;
        slots[base + src] = ss * d.ways + w;
        owner[ss * d.ways + w] = base + src;
      }
      __syncwarp();  // the entry is written before the next key of the warp reads its set
    }
  }
}

// Each key's row into its slot, unless a later key of the batch took the slot.
__global__ void cache_copy_in_kernel(ska_cache_desc d, const int32_t* counts, const int32_t* owner,
                                     const ska_cache_key* keys, const float* rows, const int32_t* slots, int n,
                                     float* data) {
  for (int i = blockIdx.x; i < n; i += gridDim.x) {
    const int slot = slots[i];
    const int s = slot / d.ways;
    if (counts[s] != 1 && owner[slot] != i) continue;
    const float4* src = reinterpret_cast<const float4*>(rows + static_cast<int64_t>(i) * d.row_floats);
    float4* dst = reinterpret_cast<float4*>(data + static_cast<int64_t>(slot) * d.row_floats);
    for (int c = threadIdx.x; c < d.row_floats / 4; c += blockDim.x) dst[c] = src[c];
  }
}

// get: one CTA per key (its first warp looks the key up), the row copied by the whole CTA.
__global__ void cache_get_kernel(ska_cache_desc d, const CacheEntry* entries, const float* data,
                                 const ska_cache_key* keys, int n, int64_t now, float* out, int32_t* hits) {
  __shared__ int found;
  for (int i = blockIdx.x; i < n; i += gridDim.x) {
    if (threadIdx.x < 32) {
      const ska_cache_key k = keys[i];
      const int s = cache_set(k, d.num_sets);
      const int lane = threadIdx.x;
      bool m = false;
      if (lane < d.ways) {
        const CacheEntry e = entries[static_cast<int64_t>(s) * d.ways + lane];
        m = same_key(e, k) && live(e, now, d.ttl);
      }
      const uint32_t b = __ballot_sync(0xffffffffu, m);
      if (lane == 0) {
        found = b ? s * d.ways + (__ffs(b) - 1) : -1;
        hits[i] = b ? 1 : 0;
      }
    }
    __syncthreads();
    const int slot = found;
    float4* dst = reinterpret_cast<float4*>(out + static_cast<int64_t>(i) * d.row_floats);
    if (slot >= 0) {
      const float4* src = reinterpret_cast<const float4*>(data + static_cast<int64_t>(slot) * d.row_floats);
      for (int c = threadIdx.x; c < d.row_floats / 4; c += blockDim.x) dst[c] = src[c];
    } else {
      for (int c = threadIdx.x; c < d.row_floats / 4; c += blockDim.x) dst[c] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    __syncthreads();
  }
}

}  // namespace

bool cache_desc_ok(const ska_cache_desc* d) {
  return d && d->num_sets >= 1 && d->num_sets <= (1 << 24) && (d->num_sets & (d->num_sets - 1)) == 0 &&
         d->ways >= 1 && d->ways <= 32 && d->row_floats >= 4 && d->row_floats % 4 == 0 && d->ttl >= 0 &&
         int64_t(d->num_sets) * d->ways <= (int64_t(1) << 30);
}

size_t cache_bytes(const ska_cache_desc& d) { return cache_layout(d).total; }

cudaError_t launch_cache_init(const ska_cache_desc& d, void* cache, cudaStream_t s) {
  const CacheLayout L = cache_layout(d);
  const int64_t slots = int64_t(d.num_sets) * d.ways;
  const int blocks = static_cast<int>(std::min<int64_t>((slots + 255) / 256, 148 * 8));
  cache_init_kernel<<<blocks, 256, 0, s>>>(reinterpret_cast<CacheEntry*>(static_cast<uint8_t*>(cache) + L.entries),
                                           slots);
  return cudaGetLastError();
}

cudaError_t launch_cache_put(const ska_cache_desc& d, void* cache, const ska_cache_key* keys, const float* rows, int n,
                             int64_t now, int32_t* slots, cudaStream_t s) {
  const CacheLayout L = cache_layout(d);
  uint8_t* c = static_cast<uint8_t*>(cache);
  CacheEntry* entries = reinterpret_cast<CacheEntry*>(c + L.entries);
  int32_t* counts = reinterpret_cast<int32_t*>(c + L.counts);
  int32_t* owner = reinterpret_cast<int32_t*>(c + L.owner);
  float* data = reinterpret_cast<float*>(c + L.data);
  cudaError_t e = cudaMemsetAsync(counts, 0, size_t(d.num_sets) * 4, s);
  if (e != cudaSuccess || n == 0) return e;
  const int blocks = std::min((n + 255) / 256, 148 * 4);
  cache_count_kernel<<<blocks, 256, 0, s>>>(keys, n, d.num_sets, counts);
  const int wblocks = std::min((n + 7) / 8, 148 * 8);  // 8 warps a block, one key a warp
  cache_put_unique_kernel<<<wblocks, 256, 0, s>>>(d, entries, counts, keys, n, now, slots);
  cache_put_shared_kernel<<<1, 32, 0, s>>>(d, entries, counts, owner, keys, n, now, slots);
  cache_copy_in_kernel<<<std::min(n, 148 * 8), 128, 0, s>>>(d, counts, owner, keys, rows, slots, n, data);
  return cudaGetLastError();
}

cudaError_t launch_cache_get(const ska_cache_desc& d, const void* cache, const ska_cache_key* keys, int n, int64_t now,
                             float* out, int32_t* hits, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  const CacheLayout L = cache_layout(d);
  const uint8_t* c = static_cast<const uint8_t*>(cache);
  cache_get_kernel<<<std::min(n, 148 * 8), 128, 0, s>>>(d, reinterpret_cast<const CacheEntry*>(c + L.entries),
                                                        reinterpret_cast<const float*>(c + L.data), keys, n, now, out,
                                                        hits);
  return cudaGetLastError();
}

}  // namespace ska
