// Stacked refinement of the sketch on sm_100a (SequenceO1 §3.3, Eq. (13)-(14)):
//   X- = LN1(X~ + X^),   X~' = LN2(X- + FFN(X-)),   FFN(U) = (swish(U W_1) * (U W_g)) W_2.
// The FFN is the SwiGLU of App. G.1 with intermediate width F = 2d (App. G.3). It is applied to
// every sketch row (b, h, j), using the weights and LayerNorm parameters of head h.
//
// One CTA of 512 threads takes 128 rows of one (user, head) at a time, four threads per row, each
// on a quarter of the columns (LayerNorm statistics combined through shared memory):
//   1. X- = LN1(x_tilde + x_hat) in fp32. The thread keeps its slice in registers for the
//      residual of step 5. It is also written to shared memory as a bf16 pair hi + lo
//      (16 significant bits) in the K-major A-operand layout. Thread 0 then prefetches the CTA's
//      next tile of x_tilde and x_hat into L2.
//   2. MMA: H1 = X- W_1 and Hg = X- W_g (M = 128, N = F, K = d; one pass for hi, one for lo),
//      accumulated in TMEM.
//   3. G = swish(H1) * Hg, again as a bf16 hi + lo pair in shared memory.
//   4. MMA: Y = G W_2 (M = 128, N = d, K = F; hi and lo passes) into the TMEM columns H1 held.
//   5. X~' = LN2(X- + Y) in fp32, written to global memory (plus a bf16 copy when asked for).
//   6. (optional) the next layer's queries X~' W_Q (Eq. (10)): X~' as a bf16 hi + lo pair in
//      shared memory, MMA against W_Q (M = 128, N = d, K = d), rounded to bf16.
// In projection mode the kernel runs step 6 alone on its input rows: the layer-0 queries
// P^(0) W_Q of Eq. (7).
// The weights are bf16 inputs. Multiplying them with the hi + lo pairs leaves about 2^-17 relative
// error per product, and the fp32 accumulation does the rest. Thread 0 issues the TMA weight
// loads and the MMAs. The phases of one tile run in sequence. The kernel is memory-bound at its
// sizes: a row reads 2d fp32 values and writes d.
//
// Weight tiles in shared memory are MN-major B operands. W_1 and W_g ([d, F], F contiguous) load
// as F/64 blocks of [d rows x 64 columns]; W_2 ([F, d], d contiguous) as d/64 blocks of
// [F rows x 64 columns].
#include <cmath>

#include "ska_internal.h"
#include "ska_ptx.cuh"

namespace ska {

namespace {

constexpr int kGroups = 4;                    // threads per row, each on a column slice
constexpr int kRefThreads = 128 * kGroups;
constexpr uint32_t kRefBlk = 16384;  // [128 rows x 64 bf16] swizzled block

template <int D, int F>
struct RefLayout {
  // Region A holds X hi | X lo during MMA1, then W_2.
  // Region B holds W_1 | W_g during MMA1, then G hi | G lo.
  static constexpr uint32_t x_bytes = (D / 64) * kRefBlk;
  static constexpr uint32_t g_bytes = (F / 64) * kRefBlk;
  static constexpr uint32_t w_bytes = D * F * 2;
  static constexpr uint32_t wq_bytes = D * D * 2;
  static constexpr uint32_t a_bytes = (2 * x_bytes > w_bytes) ? 2 * x_bytes : w_bytes;
  static constexpr uint32_t b_bytes = (2 * g_bytes > 2 * w_bytes) ? 2 * g_bytes : 2 * w_bytes;
  static constexpr uint32_t x_hi = 0;
  static constexpr uint32_t x_lo = x_bytes;
  static constexpr uint32_t w2 = 0;
  static constexpr uint32_t w1 = a_bytes;
  static constexpr uint32_t wg = a_bytes + w_bytes;
  static constexpr uint32_t g_hi = a_bytes;
  static constexpr uint32_t g_lo = a_bytes + g_bytes;
  static constexpr uint32_t red = a_bytes + b_bytes;         // kGroups x 128 partial row sums
  static constexpr uint32_t bars = red + kGroups * 128 * 4;
  static constexpr uint32_t total = bars + 128;
  static_assert(a_bytes % 1024 == 0 && w_bytes % 1024 == 0 && g_bytes % 1024 == 0, "1024-byte aligned blocks");
  static_assert(total <= 227 * 1024, "fits in shared memory");
  static_assert(wq_bytes <= b_bytes, "W_Q fits in region B");
};

struct RefBars {
  uint64_t w1g, w2, x, m1, g, m2, wq, xq, m3, drain;
  uint32_t tmem_base;
  int abort_flag;
};

struct RefWaiter {
  RefBars* bars;
  int* status;
  uint64_t budget;
  // Bounded wait. A wait that runs out records SKA_ERR_DEVICE_TIMEOUT and raises the CTA's abort
  // flag, after which the other waits give up at once (drain waits still run to their limit).
  __device__ __forceinline__ bool operator()(uint64_t* bar, uint32_t parity, bool drain = false) {
    volatile int* ab = &bars->abort_flag;
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
      if (mbar_try_wait(bar, parity)) return true;
      if (!drain && *ab) return false;
      if (globaltimer_ns() - t0 > budget) {
        atomicCAS(status, 0, (int)SKA_ERR_DEVICE_TIMEOUT);
        *ab = 1;
        return false;
      }
    }
  }
};

// Splits 8 fp32 values into a bf16 hi + lo pair (lo = bf16(v - hi)) and stores them at row r,
// columns c .. c + 7, of two swizzled K-major operands.
__device__ __forceinline__ void store_pair8(uint8_t* hi, uint8_t* lo, int r, int c, const float* v) {
  float h[8], l[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    h[u] = __bfloat162float(__float2bfloat16_rn(v[u]));
    l[u] = v[u] - h[u];
  }
  const uint32_t off = (c >> 6) * kRefBlk + sw128_offset(r, (c & 63) * 2);
  *reinterpret_cast<uint4*>(hi + off) =
      make_uint4(pack_bf16x2(h[0], h[1]), pack_bf16x2(h[2], h[3]), pack_bf16x2(h[4], h[5]), pack_bf16x2(h[6], h[7]));
  *reinterpret_cast<uint4*>(lo + off) =
      make_uint4(pack_bf16x2(l[0], l[1]), pack_bf16x2(l[2], l[3]), pack_bf16x2(l[4], l[5]), pack_bf16x2(l[6], l[7]));
}

// LayerNorm of one row held by one thread: mean, biased variance (two passes), normalisation,
// then the affine map (gamma, beta may be null: 1 and 0) in float4 steps.
template <int D>
__device__ __forceinline__ void layer_norm_row(float* x, const float* gamma, const float* beta, float eps) {
  float mean = 0.f;
#pragma unroll
  for (int c = 0; c < D; ++c) mean += x[c];
  mean *= 1.f / D;
  float var = 0.f;
#pragma unroll
  for (int c = 0; c < D; ++c) {
    const float t = x[c] - mean;
    var = fmaf(t, t, var);
  }
  const float rs = rsqrtf(var * (1.f / D) + eps);
#pragma unroll
  for (int c = 0; c < D; ++c) x[c] = (x[c] - mean) * rs;
  if (gamma) {
    const float4* g4 = reinterpret_cast<const float4*>(gamma);
#pragma unroll
    for (int u = 0; u < D / 4; ++u) {
      const float4 g = __ldg(g4 + u);
      x[4 * u] *= g.x;
      x[4 * u + 1] *= g.y;
      x[4 * u + 2] *= g.z;
      x[4 * u + 3] *= g.w;
    }
  }
  if (beta) {
    const float4* b4 = reinterpret_cast<const float4*>(beta);
#pragma unroll
    for (int u = 0; u < D / 4; ++u) {
      const float4 b = __ldg(b4 + u);
      x[4 * u] += b.x;
      x[4 * u + 1] += b.y;
      x[4 * u + 2] += b.z;
      x[4 * u + 3] += b.w;
    }
  }
}

template <int D>
__device__ __forceinline__ void store_row_f32(float* dst, const float* x) {
  float4* o = reinterpret_cast<float4*>(dst);
#pragma unroll
  for (int u = 0; u < D / 4; ++u) o[u] = make_float4(x[4 * u], x[4 * u + 1], x[4 * u + 2], x[4 * u + 3]);
}

template <int D>
__device__ __forceinline__ void store_row_bf16(uint8_t* dst, const float* x) {
  uint4* ob = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int u = 0; u < D / 8; ++u)
    ob[u] = make_uint4(pack_bf16x2(x[8 * u], x[8 * u + 1]), pack_bf16x2(x[8 * u + 2], x[8 * u + 3]),
                       pack_bf16x2(x[8 * u + 4], x[8 * u + 5]), pack_bf16x2(x[8 * u + 6], x[8 * u + 7]));
}

// Row statistics of a LayerNorm whose row is split over the kGroups threads of one TMEM lane: each
// passes its partial sum and receives the row's total through shared memory (CTA barriers: every
// thread of the CTA calls this at the same point).
__device__ __forceinline__ float row_total(float part, float* red, int grp, int r) {
  red[grp * 128 + r] = part;
  __syncthreads();
  float t = 0.f;
#pragma unroll
  for (int g = 0; g < kGroups; ++g) t += red[g * 128 + r];
  __syncthreads();  // the slots are free for the next use
  return t;
}

// LayerNorm of a row held as kGroups slices of C values (this thread: columns [c0, c0 + C)); the
// statistics are over the whole row of D values, in two passes (mean, then squared deviations).
template <int C, int D>
__device__ __forceinline__ void layer_norm_slice(float* x, int c0, const float* gamma, const float* beta, float eps,
                                                 float* red, int grp, int r) {
  float s = 0.f;
#pragma unroll
  for (int c = 0; c < C; ++c) s += x[c];
  const float mean = row_total(s, red, grp, r) * (1.f / D);
  float v = 0.f;
#pragma unroll
  for (int c = 0; c < C; ++c) {
    const float t = x[c] - mean;
    v = fmaf(t, t, v);
  }
  const float rs = rsqrtf(row_total(v, red, grp, r) * (1.f / D) + eps);
#pragma unroll
  for (int c = 0; c < C; ++c) x[c] = (x[c] - mean) * rs;
  if (gamma) {
    const float4* g4 = reinterpret_cast<const float4*>(gamma + c0);
#pragma unroll
    for (int u = 0; u < C / 4; ++u) {
      const float4 g = __ldg(g4 + u);
      x[4 * u] *= g.x;
      x[4 * u + 1] *= g.y;
      x[4 * u + 2] *= g.z;
      x[4 * u + 3] *= g.w;
    }
  }
  if (beta) {
    const float4* b4 = reinterpret_cast<const float4*>(beta + c0);
#pragma unroll
    for (int u = 0; u < C / 4; ++u) {
      const float4 b = __ldg(b4 + u);
      x[4 * u] += b.x;
      x[4 * u + 1] += b.y;
      x[4 * u + 2] += b.z;
      x[4 * u + 3] += b.w;
    }
  }
}

template <int C>
__device__ __forceinline__ void load_slice(const float* src, float* x) {
  const float4* a = reinterpret_cast<const float4*>(src);
#pragma unroll
  for (int u = 0; u < C / 4; ++u) {
    const float4 v = a[u];
    x[4 * u] = v.x;
    x[4 * u + 1] = v.y;
    x[4 * u + 2] = v.z;
    x[4 * u + 3] = v.w;
  }
}

template <int D, int F>
__global__ void __launch_bounds__(kRefThreads, 1)
    sa_refine_kernel(const __grid_constant__ CUtensorMap mapW1, const __grid_constant__ CUtensorMap mapWg,
                     const __grid_constant__ CUtensorMap mapW2, const __grid_constant__ CUtensorMap mapWq,
                     const RefineParams p) {
  using L = RefLayout<D, F>;
  constexpr uint32_t kCols = 2 * F;  // H1 | Hg
  constexpr int XC = D / kGroups;    // columns of X, Y and q per thread
  constexpr int GC = F / kGroups;    // columns of G per thread
  static_assert(kCols <= 512 && (kCols & (kCols - 1)) == 0, "TMEM allocation is a power of two <= 512");
  static_assert(XC % 16 == 0 && GC % 32 == 0, "column slices");
  extern __shared__ __align__(1024) uint8_t smem[];
  RefBars& bars = *reinterpret_cast<RefBars*>(smem + L::bars);
  float* red = reinterpret_cast<float*>(smem + L::red);
  if ((smem_u32(smem) & 1023u) != 0) {
    if (threadIdx.x == 0) atomicCAS(p.status, 0, (int)SKA_ERR_UNSUPPORTED);
    return;
  }
  const int warp = threadIdx.x >> 5;
  const int r = threadIdx.x & 127;  // the row (TMEM lane) of this thread
  const int grp = warp >> 2;        // its column slice
  const bool ctl = (threadIdx.x == 0);
  constexpr uint32_t kArrivals = kRefThreads / 32;
  if (ctl) {
    mbar_init(&bars.w1g, 1);
    mbar_init(&bars.w2, 1);
    mbar_init(&bars.x, kArrivals);
    mbar_init(&bars.m1, 1);
    mbar_init(&bars.g, kArrivals);
    mbar_init(&bars.m2, 1);
    mbar_init(&bars.wq, 1);
    mbar_init(&bars.xq, kArrivals);
    mbar_init(&bars.m3, 1);
    mbar_init(&bars.drain, 1);
    bars.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&bars.tmem_base, kCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = bars.tmem_base;
  const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
  RefWaiter wait{&bars, p.status, p.budget_ns};
  uint8_t* sXh = smem + L::x_hi;
  uint8_t* sXl = smem + L::x_lo;
  uint8_t* sW1 = smem + L::w1;
  uint8_t* sWg = smem + L::wg;
  uint8_t* sW2 = smem + L::w2;
  uint8_t* sGh = smem + L::g_hi;
  uint8_t* sGl = smem + L::g_lo;
  uint8_t* sWq = sW1;  // W_Q into region B once G has been read
  constexpr uint32_t i1 = idesc_bf16_f32(128, F, false, true);
  constexpr uint32_t i2 = idesc_bf16_f32(128, D, false, true);
  const int tiles_per_bh = (p.k + 127) / 128;
  const int ntiles = p.B * p.H * tiles_per_bh;
  const int xc0 = grp * XC, gc0 = grp * GC;
  int it = 0;
  bool w1g_pending = false, w2_pending = false, wq_pending = false;  // thread 0: loads not yet waited for
  const bool project_only = p.mode == 1;
  // thread 0: W_Q of head h into region B
  auto load_wq = [&](int h) {
    mbar_expect_tx(&bars.wq, L::wq_bytes);
    for (int nb = 0; nb < D / 64; ++nb) tma_load_2d(sWq + nb * D * 128, &mapWq, &bars.wq, nb * 64, h * D);
    wq_pending = true;
  };
  // this thread's slice of the rows to project, as a bf16 hi + lo pair in region A, then the
  // warp's arrival on xq
  auto stage_x = [&](const float* x) {
#pragma unroll
    for (int c = 0; c < XC; c += 8) store_pair8(sXh, sXl, r, xc0 + c, x + c);
    fence_async_shared();
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(&bars.xq);
  };
  // tiles in (h, b, row tile) order
  for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++it) {
    const int h = tile / (p.B * tiles_per_bh);
    const int rem = tile - h * p.B * tiles_per_bh;
    const int b = rem / tiles_per_bh;
    const int j = (rem - b * tiles_per_bh) * 128 + r;
    const bool valid = j < p.k;
    const int64_t row = (static_cast<int64_t>(b) * p.H + h) * p.k + j;
    const int64_t xrow = p.x_tilde_shared ? static_cast<int64_t>(h) * p.k + j : row;
    const uint32_t par = it & 1;
    bool ok = true;
    float xb[XC];
    if (project_only) {
      if (ctl) load_wq(h);
      if (valid) {
        load_slice<XC>(p.x_tilde + xrow * D + xc0, xb);
      } else {
#pragma unroll
        for (int u = 0; u < XC; ++u) xb[u] = 0.f;
      }
      stage_x(xb);
    } else {
      if (ctl) {  // W_1, W_g of head h into region B (the previous tile's MMAs have all completed)
        mbar_expect_tx(&bars.w1g, 2 * L::w_bytes);
        for (int nb = 0; nb < F / 64; ++nb) {
          tma_load_2d(sW1 + nb * D * 128, &mapW1, &bars.w1g, nb * 64, h * D);
          tma_load_2d(sWg + nb * D * 128, &mapWg, &bars.w1g, nb * 64, h * D);
        }
        w1g_pending = true;
      }
      // 1. X- = LN1(x_tilde + x_hat)
      if (valid) {
        float xh[XC];
        load_slice<XC>(p.x_tilde + xrow * D + xc0, xb);
        load_slice<XC>(p.x_hat + row * D + xc0, xh);
#pragma unroll
        for (int u = 0; u < XC; ++u) xb[u] += xh[u];
      } else {
#pragma unroll
        for (int u = 0; u < XC; ++u) xb[u] = 0.f;
      }
      layer_norm_slice<XC, D>(xb, xc0, p.gamma1 ? p.gamma1 + h * D : nullptr, p.beta1 ? p.beta1 + h * D : nullptr,
                              p.eps, red, grp, r);
      if (valid) {
        if (p.x_bar) store_row_f32<XC>(p.x_bar + row * D + xc0, xb);
      } else {
#pragma unroll
        for (int u = 0; u < XC; ++u) xb[u] = 0.f;
      }
#pragma unroll
      for (int c = 0; c < XC; c += 8) store_pair8(sXh, sXl, r, xc0 + c, xb + c);
      fence_async_shared();
      __syncwarp();
      if ((threadIdx.x & 31) == 0) mbar_arrive(&bars.x);
      if (ctl && tile + static_cast<int>(gridDim.x) < ntiles) {
        // the next tile's rows of x_tilde and x_hat into L2 while this tile computes
        const int nt = tile + gridDim.x;
        const int nh = nt / (p.B * tiles_per_bh), nrem = nt - nh * p.B * tiles_per_bh;
        const int nb = nrem / tiles_per_bh, nj0 = (nrem - nb * tiles_per_bh) * 128;
        const uint32_t bytes = static_cast<uint32_t>(min(128, p.k - nj0)) * D * 4;
        const int64_t nrow = (static_cast<int64_t>(nb) * p.H + nh) * p.k + nj0;
        const int64_t nxrow = p.x_tilde_shared ? static_cast<int64_t>(nh) * p.k + nj0 : nrow;
        bulk_prefetch_l2(p.x_tilde + nxrow * D, bytes);
        bulk_prefetch_l2(p.x_hat + nrow * D, bytes);
      }
      // 2. H1 = X- W_1, Hg = X- W_g
      if (ctl) {
        ok = wait(&bars.x, par) && wait(&bars.w1g, par);
        if (ok) {
          w1g_pending = false;
          tc_fence_after();
#pragma unroll 1
          for (int half = 0; half < 2; ++half) {
            const uint32_t xa = smem_u32(half ? sXl : sXh);
#pragma unroll
            for (int s = 0; s < D / 16; ++s) {
              const uint64_t ad = sw128_desc(xa + (s / 4) * kRefBlk + (s % 4) * 32, 16, 1024);
              const uint32_t acc = (half | s) > 0;
              umma_bf16(tb, ad, sw128_desc(smem_u32(sW1) + s * 2048, D * 128, 1024), i1, acc);
              umma_bf16(tb + F, ad, sw128_desc(smem_u32(sWg) + s * 2048, D * 128, 1024), i1, acc);
            }
          }
          if (!(p.debug_flags & 2u)) umma_commit(&bars.m1);  // the test hook withholds it
        }
      }
      if (!__syncthreads_and(ok && wait(&bars.m1, par))) break;
      tc_fence_after();
      if (ctl) {  // W_2 into region A, whose X hi / lo MMA1 has finished reading
        mbar_expect_tx(&bars.w2, L::w_bytes);
        for (int nb = 0; nb < D / 64; ++nb) tma_load_2d(sW2 + nb * F * 128, &mapW2, &bars.w2, nb * 64, h * F);
        w2_pending = true;
      }
      // 3. G = swish(H1) * Hg into region B (W_1 / W_g are no longer read), this thread's slice
#pragma unroll 1
      for (int c = gc0; c < gc0 + GC; c += 16) {  // (16 columns at a time: X- stays in registers)
        uint32_t v1[16], vg[16];
        tmem_ld16(tb + lane_off + c, v1);
        tmem_ld16(tb + lane_off + F + c, vg);
        tmem_ld_wait();
#pragma unroll
        for (int u = 0; u < 16; u += 8) {
          float gv[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float a = __uint_as_float(v1[u + e]);
            // swish(a) = a / (1 + e^-a); the fast divide returns -0 for a < -88 (e^-a = inf)
            gv[e] = valid ? __fdividef(a, 1.f + __expf(-a)) * __uint_as_float(vg[u + e]) : 0.f;
          }
          store_pair8(sGh, sGl, r, c + u, gv);
        }
      }
      fence_async_shared();
      tc_fence_before();
      __syncwarp();
      if ((threadIdx.x & 31) == 0) mbar_arrive(&bars.g);
      // 4. Y = G W_2 into TMEM columns [0, D)
      if (ctl) {
        ok = wait(&bars.g, par) && wait(&bars.w2, par);
        if (ok) {
          w2_pending = false;
          tc_fence_after();
#pragma unroll 1
          for (int half = 0; half < 2; ++half) {
            const uint32_t ga = smem_u32(half ? sGl : sGh);
#pragma unroll
            for (int s = 0; s < F / 16; ++s)
              umma_bf16(tb, sw128_desc(ga + (s / 4) * kRefBlk + (s % 4) * 32, 16, 1024),
                        sw128_desc(smem_u32(sW2) + s * 2048, F * 128, 1024), i2, (half | s) > 0);
          }
          umma_commit(&bars.m2);
        }
      }
      if (!__syncthreads_and(ok && wait(&bars.m2, par))) break;
      tc_fence_after();
      if (ctl && p.q_next) load_wq(h);  // region B is free: MMA2 has read G
      // 5. X~' = LN2(X- + Y), X- still in xb (zero on rows past k)
#pragma unroll
      for (int c = 0; c < XC; c += 16) {
        uint32_t yv[16];
        tmem_ld16(tb + lane_off + xc0 + c, yv);
        tmem_ld_wait();
#pragma unroll
        for (int u = 0; u < 16; ++u) xb[c + u] += __uint_as_float(yv[u]);
      }
      tc_fence_before();
      layer_norm_slice<XC, D>(xb, xc0, p.gamma2 ? p.gamma2 + h * D : nullptr, p.beta2 ? p.beta2 + h * D : nullptr,
                              p.eps, red, grp, r);
      if (valid) {
        store_row_f32<XC>(p.x_next + row * D + xc0, xb);
        if (p.x_next_bf16) store_row_bf16<XC>(p.x_next_bf16 + (row * D + xc0) * 2, xb);
      } else {
#pragma unroll
        for (int u = 0; u < XC; ++u) xb[u] = 0.f;
      }
      if (p.q_next) stage_x(xb);  // region A: W_2 there has been read by MMA2
    }  // full refinement
    if (p.q_next) {
      // 6. the next layer's queries: X~' W_Q from the hi + lo pair staged in region A
      if (ctl) {
        ok = wait(&bars.xq, par) && wait(&bars.wq, par);
        if (ok) {
          wq_pending = false;
          tc_fence_after();
#pragma unroll 1
          for (int half = 0; half < 2; ++half) {
            const uint32_t xa = smem_u32(half ? sXl : sXh);
#pragma unroll
            for (int s = 0; s < D / 16; ++s)
              umma_bf16(tb, sw128_desc(xa + (s / 4) * kRefBlk + (s % 4) * 32, 16, 1024),
                        sw128_desc(smem_u32(sWq) + s * 2048, D * 128, 1024), i2, (half | s) > 0);
          }
          umma_commit(&bars.m3);
        }
      }
      if (!__syncthreads_and(ok && wait(&bars.m3, par))) break;
      tc_fence_after();
      uint4* qo = reinterpret_cast<uint4*>(p.q_next + (row * D + xc0) * 2);
#pragma unroll
      for (int c = 0; c < XC; c += 16) {
        uint32_t qv[16];
        tmem_ld16(tb + lane_off + xc0 + c, qv);
        tmem_ld_wait();
        if (valid) {
#pragma unroll
          for (int u = 0; u < 16; u += 8)
            qo[(c + u) / 8] = make_uint4(pack_bf16x2(__uint_as_float(qv[u]), __uint_as_float(qv[u + 1])),
                                         pack_bf16x2(__uint_as_float(qv[u + 2]), __uint_as_float(qv[u + 3])),
                                         pack_bf16x2(__uint_as_float(qv[u + 4]), __uint_as_float(qv[u + 5])),
                                         pack_bf16x2(__uint_as_float(qv[u + 6]), __uint_as_float(qv[u + 7])));
        }
      }
      tc_fence_before();
    }
    __syncthreads();  // every thread is done with this tile's TMEM and shared memory
  }
  if (ctl) {
    // all issued MMAs, and any weight load a stopped tile left in flight, end before the exit
    umma_commit(&bars.drain);
    wait(&bars.drain, 0, true);
    if (w1g_pending) wait(&bars.w1g, it & 1, true);
    if (w2_pending) wait(&bars.w2, it & 1, true);
    if (wq_pending) wait(&bars.wq, it & 1, true);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tb, kCols);
  }
}

// After a device-side error, every output element becomes NaN (the rows the stopped CTAs did not
// reach would otherwise hold stale values).
__global__ void refine_poison_kernel(const int* status, float* x_next, float* x_bar, uint16_t* x_next_bf16,
                                     uint16_t* q_next, int64_t n) {
  if (*reinterpret_cast<const volatile int*>(status) == 0) return;
  const float nan = __int_as_float(0x7fc00000);
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x) {
    if (x_next) x_next[i] = nan;
    if (x_bar) x_bar[i] = nan;
    if (x_next_bf16) x_next_bf16[i] = 0x7fc0;
    if (q_next) q_next[i] = 0x7fc0;
  }
}

template <int D, int F>
cudaError_t refine_launch_t(int num_ctas, const CUtensorMap& m1, const CUtensorMap& mg, const CUtensorMap& m2,
                            const CUtensorMap& mq, const RefineParams& p, cudaStream_t stream) {
  auto kern = sa_refine_kernel<D, F>;
  const size_t smem = RefLayout<D, F>::total;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<num_ctas, kRefThreads, smem, stream>>>(m1, mg, m2, mq, p);
  return cudaGetLastError();
}

}  // namespace

bool sa_refine_supported(int D, int F) { return (D == 64 && F == 128) || (D == 128 && F == 256); }

cudaError_t launch_sa_refine(int D, int F, int num_ctas, const CUtensorMap& m1, const CUtensorMap& mg,
                             const CUtensorMap& m2, const CUtensorMap& mq, const RefineParams& p,
                             cudaStream_t stream) {
  cudaError_t e = cudaErrorInvalidValue;
  if (D == 64 && F == 128) e = refine_launch_t<64, 128>(num_ctas, m1, mg, m2, mq, p, stream);
  if (D == 128 && F == 256) e = refine_launch_t<128, 256>(num_ctas, m1, mg, m2, mq, p, stream);
  return e;
}

cudaError_t launch_refine_poison(int D, const RefineParams& p, cudaStream_t stream) {
  const int64_t n = int64_t(p.B) * p.H * p.k * D;
  refine_poison_kernel<<<2 * 148, 256, 0, stream>>>(p.status, p.x_next, p.x_bar,
                                                    reinterpret_cast<uint16_t*>(p.x_next_bf16),
                                                    reinterpret_cast<uint16_t*>(p.q_next), n);
  return cudaGetLastError();
}

}  // namespace ska
