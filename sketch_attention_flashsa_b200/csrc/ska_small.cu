// Small SIMT kernels around the fused SA kernels: tile scheduling from cu_seqlens, the
// fixed-order combine of per-cluster partial sketches, -inf padding of the per-token lse,
// and the fp32 -> bf16 input conversion.
#include <algorithm>

#include <cuda_bf16.h>

#include "ska_internal.h"

namespace ska {

namespace {

__device__ __forceinline__ int used_len(const int32_t* cu, const int32_t* seqused, int b) {
  int len = cu[b + 1] - cu[b];
  if (seqused) len = min(len, seqused[b]);
  return max(len, 0);
}

// One block. tile_prefix[b] = sum_{b' < b} ceil(used_b' / 128); header gets the stream size and
// the number of tiles each persistent cluster takes. Also clears the device status word.
__global__ void __launch_bounds__(1024) schedule_kernel(const int32_t* __restrict__ cu,
                                                        const int32_t* __restrict__ seqused, int B, int H,
                                                        int num_clusters, int32_t* __restrict__ prefix,
                                                        WsHeader* hdr) {
  __shared__ int part[1024];
  const int t = threadIdx.x;
  const int per = (B + 1023) / 1024;
  const int lo = min(B, t * per), hi = min(B, lo + per);
  int s = 0;
  for (int b = lo; b < hi; ++b) s += (used_len(cu, seqused, b) + kTileTokens - 1) / kTileTokens;
  part[t] = s;
  __syncthreads();
  // inclusive scan of the 1024 partial sums (Hillis-Steele)
  for (int off = 1; off < 1024; off <<= 1) {
    int v = (t >= off) ? part[t - off] : 0;
    __syncthreads();
    part[t] += v;
    __syncthreads();
  }
  int run = (t == 0) ? 0 : part[t - 1];
  for (int b = lo; b < hi; ++b) {
    prefix[b] = run;
    run += (used_len(cu, seqused, b) + kTileTokens - 1) / kTileTokens;
  }
  if (t == 1023) {
    prefix[B] = part[1023];
    // the host bounds H * (tiles) below 2^31 (descriptor check); 64-bit here all the same
    const long long total = static_cast<long long>(H) * part[1023];
    hdr->total_tiles = static_cast<int>(total);
    hdr->tiles_per_cluster = static_cast<int>((total + num_clusters - 1) / num_clusters);
    hdr->status = 0;
  }
}

// sketch[s, :, :] = sum over the clusters p that touched segment s of partial[s + p, :, :],
// in increasing p. Segment s = b*H + h covers global tiles [H*prefix[b] + h*n_b, ... + n_b).
// When an earlier kernel of the call recorded an error the outputs are NaN; a sum that is not
// finite (a value row that overflowed fp16 once scaled by its weight) is recorded as
// SKA_ERR_RANGE.
__global__ void proto_combine_kernel(const int32_t* __restrict__ prefix, WsHeader* __restrict__ hdr,
                                     const float* __restrict__ partial, const float* __restrict__ mass_partial,
                                     int B, int H, int k, int D, float* __restrict__ sketch,
                                     float* __restrict__ mass, bool renormalize) {
  const int s = blockIdx.x;
  const bool failed = *reinterpret_cast<volatile int32_t*>(&hdr->status) != 0;
  bool finite = true;
  const int b = s / H, h = s - b * H;
  const int nb = prefix[b + 1] - prefix[b];
  const int W = hdr->tiles_per_cluster;
  const int64_t per = static_cast<int64_t>(k) * D;
  int p0 = 0, p1 = -1;
  if (nb > 0 && W > 0) {
    const int t0 = H * prefix[b] + h * nb;
    p0 = t0 / W;
    p1 = (t0 + nb - 1) / W;
  }
  for (int64_t e = (static_cast<int64_t>(blockIdx.y) * blockDim.x + threadIdx.x) * 4; e < per;
       e += static_cast<int64_t>(gridDim.y) * blockDim.x * 4) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int pc = p0; pc <= p1; ++pc) {
      const float4 v = *reinterpret_cast<const float4*>(partial + (static_cast<int64_t>(s + pc) * per + e));
      acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
    }
    finite = finite && isfinite(acc.x) && isfinite(acc.y) && isfinite(acc.z) && isfinite(acc.w);
    if (renormalize) {
      // the prototype's mass, summed in the same order as its mass output
      const int j = static_cast<int>(e / D);
      float mj = 0.f;
      for (int pc = p0; pc <= p1; ++pc) mj += mass_partial[static_cast<int64_t>(s + pc) * k + j];
      const float inv = mj > 0.f ? 1.f / mj : 0.f;
      acc.x *= inv; acc.y *= inv; acc.z *= inv; acc.w *= inv;
    }
    if (failed) acc = make_float4(NAN, NAN, NAN, NAN);
    *reinterpret_cast<float4*>(sketch + static_cast<int64_t>(s) * per + e) = acc;
  }
  if (mass && blockIdx.y == 0) {
    for (int j = threadIdx.x; j < k; j += blockDim.x) {
      float acc = 0.f;
      for (int pc = p0; pc <= p1; ++pc) acc += mass_partial[static_cast<int64_t>(s + pc) * k + j];
      finite = finite && isfinite(acc);
      mass[static_cast<int64_t>(s) * k + j] = failed ? NAN : acc;
    }
  }
  if (!finite && !failed) atomicCAS(&hdr->status, 0, static_cast<int>(SKA_ERR_RANGE));
}

// lse rows of padding tokens (positions >= seqused[b] inside user b) are -inf, their maximum
// weights -1.
__global__ void fill_padding_lse_kernel(const int32_t* __restrict__ cu, const int32_t* __restrict__ seqused,
                                        int B, int H, int64_t T, float* __restrict__ lse, float* __restrict__ maxw) {
  const int b = blockIdx.x;
  if (b >= B) return;
  const int64_t lo = cu[b] + used_len(cu, seqused, b);
  const int64_t hi = (static_cast<int64_t>(cu[b + 1]) < T) ? static_cast<int64_t>(cu[b + 1]) : T;
  if (hi <= lo) return;
  const int64_t n = static_cast<int64_t>(hi - lo) * H;
  for (int64_t i = threadIdx.x; i < n; i += blockDim.x) {
    if (lse) lse[lo * H + i] = -INFINITY;
    if (maxw) maxw[lo * H + i] = -1.f;
  }
}

// Histogram of values in [0, 1]: per-block counts in shared memory, then added into the global
// counts (integer additions: the result does not depend on their order).
__global__ void weight_histogram_kernel(const float* __restrict__ v, int64_t n, int bins, int32_t* __restrict__ counts) {
  extern __shared__ int32_t local[];
  for (int b = threadIdx.x; b < bins; b += blockDim.x) local[b] = 0;
  __syncthreads();
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float x = v[i];
    if (!(x >= 0.f)) continue;  // padding (-1) and NaN
    const int b = min(static_cast<int>(x * bins), bins - 1);
    atomicAdd(&local[b], 1);
  }
  __syncthreads();
  for (int b = threadIdx.x; b < bins; b += blockDim.x)
    if (local[b]) atomicAdd(&counts[b], local[b]);
}

__global__ void cast_f32_bf16_kernel(const float* __restrict__ src, __nv_bfloat16* __restrict__ dst, int64_t n) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    dst[i] = __float2bfloat16_rn(src[i]);
}

}  // namespace

cudaError_t launch_schedule(const int32_t* cu, const int32_t* seqused, int B, int H, int num_clusters,
                            int32_t* prefix, WsHeader* hdr, cudaStream_t stream) {
  schedule_kernel<<<1, 1024, 0, stream>>>(cu, seqused, B, H, num_clusters, prefix, hdr);
  return cudaGetLastError();
}

cudaError_t launch_proto_combine(const int32_t* prefix, WsHeader* hdr, const float* partial,
                                 const float* mass_partial, int B, int H, int k, int D, float* sketch,
                                 float* mass, bool renormalize, cudaStream_t stream) {
  const int per4 = (k * D) / 4;
  const int threads = 256;
  const int bx = std::min(32, (per4 + threads - 1) / threads);
  dim3 grid(B * H, bx, 1);
  proto_combine_kernel<<<grid, threads, 0, stream>>>(prefix, hdr, partial, mass_partial, B, H, k, D, sketch, mass,
                                                     renormalize);
  return cudaGetLastError();
}

cudaError_t launch_fill_padding_lse(const int32_t* cu, const int32_t* seqused, int B, int H, int64_t T,
                                    float* lse, float* maxw, cudaStream_t stream) {
  fill_padding_lse_kernel<<<B, 256, 0, stream>>>(cu, seqused, B, H, T, lse, maxw);
  return cudaGetLastError();
}

cudaError_t launch_weight_histogram(const float* values, int64_t n, int bins, int32_t* counts, cudaStream_t stream) {
  cudaError_t e = cudaMemsetAsync(counts, 0, size_t(bins) * sizeof(int32_t), stream);
  if (e != cudaSuccess || n == 0) return e;
  const int64_t blocks = std::min<int64_t>((n + 255) / 256, 148 * 4);
  weight_histogram_kernel<<<static_cast<unsigned>(blocks), 256, size_t(bins) * sizeof(int32_t), stream>>>(
      values, n, bins, counts);
  return cudaGetLastError();
}

cudaError_t launch_cast_f32_bf16(const float* src, void* dst, int64_t n, cudaStream_t stream) {
  if (n == 0) return cudaSuccess;
  const int threads = 256;
  const int64_t blocks = std::min<int64_t>((n + threads - 1) / threads, 148 * 16);
  cast_f32_bf16_kernel<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(
      src, static_cast<__nv_bfloat16*>(dst), n);
  return cudaGetLastError();
}

}  // namespace ska
