// STCA backward on sm_100a: gradients of <dO, out> through the target attention of SequenceO1 §2.3
// (applied to the recent suffix and the sketch in §3.4, targets of one user batched by MRLB §4.2).
// For target t of user b and head h, with keys K_t = [the first target_kv_len[t] suffix rows of b ;
// b's sketch rows], values V_t, p = softmax(scale K_t q_t) (saved as its lse) and out_t = p V_t:
//   dV_t += p dO_t,   dp = V_t dO_t,   ds = p (dp - delta_t),   delta_t = <dO_t, out_t>,
//   dq_t = scale ds K_t,   dK_t += scale ds q_t.
// Key and value gradients of rows shared by a user's targets are sums over those targets.
//
// Two kernels, so that no gradient needs atomics:
//   key-major (dK, dV): a CTA takes one 128-key tile of one (user, head) and walks the user's
//     128-target tiles:  S^T = K Q^T and dP^T = V dO^T (M = keys, N = targets, K = d) into TMEM;
//     thread = key row: P^T = 2^(scale log2e s - lse2_t), masked, and dS^T = P^T (dP^T - delta_t),
//     both as bf16 pairs written back over the first 64 columns of their own fp32 tiles;
//     dV += P^T dO and dK += dS^T Q (M = keys, N = d, K = targets), A operands read from TMEM.
//   query-major (dq): a CTA takes one 128-target tile and walks the user's key tiles: S = Q K^T,
//     dP = dO V^T; thread = target row: P, dS = P (dP - delta) split into bf16 hi + lo (hi over S,
//     lo over dP); dq += dS_hi K + dS_lo K in TMEM, restarted every kDqChain key tiles and added
//     into the output row in fp32 (the tensor core's fp32 accumulation is not round-to-nearest).
// Warps 0-15 do the row work, four warps per TMEM lane quarter, each on a group of 32 of the 128
// columns (its bf16 pairs go over the first half of its own columns, so the groups never overwrite
// each other's unread values; the MMAs read the A operand from all groups). Warp 16 lane 0 issues the
// TMA loads, warp 17 lane 0 the MMAs. Operands that stay for a whole item (K/V, or Q/dO) and the streamed ones
// are double-buffered where shared memory allows (d = 64; d = 128 keeps one item stage).
#include <algorithm>
#include <climits>
#include <cmath>

#include "ska_internal.h"
#include "ska_ptx.cuh"

namespace ska {

namespace {

constexpr int kGroups = 4;               // column groups of the row work
constexpr int kCw = 128 / kGroups;        // columns per group
constexpr int kRowWarps = 4 * kGroups;
constexpr int kSbThreads = 32 * (kRowWarps + 2);
constexpr int kProdWarp = kRowWarps, kMmaWarp = kRowWarps + 1;
constexpr uint32_t kSbBlk = 16384;  // [128 rows x 64 bf16] swizzled block
constexpr int kDqChain = 16;        // key tiles per dq accumulation chain in TMEM
constexpr float kLog2e = 1.4426950408889634f;

struct SbBars {
  uint64_t ifull[2], iempty[2];  // item operands (K/V or Q/dO)
  uint64_t sfull2[2], sempty2[2];  // streamed operands (Q/dO or K/V)
  uint64_t sfull, pfull, ofull, ofree, drain;
  uint64_t mready[2];  // key-major kernel: a target tile's values staged by the four row warps
  uint32_t tmem_base;
  int abort_flag;
};

struct SbWaiter {
  SbBars* bars;
  int* status;
  uint64_t budget;
  // Bounded wait; a wait that runs out records SKA_ERR_DEVICE_TIMEOUT and raises the abort flag,
  // after which the other waits give up at once (drain waits still run to their limit).
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

// ------------------------------------------------------------------ per-user geometry
__device__ __forceinline__ int sb_suffix(const StcaBwdParams& p, int b) { return max(p.cu_k[b + 1] - p.cu_k[b], 0); }
__device__ __forceinline__ int sb_targets(const StcaBwdParams& p, int b) { return max(p.cu_q[b + 1] - p.cu_q[b], 0); }
__device__ __forceinline__ int sb_hist_tiles(const StcaBwdParams& p, int b) { return (sb_suffix(p, b) + 127) / 128; }
__device__ __forceinline__ int sb_key_tiles(const StcaBwdParams& p, int b) {
  return sb_hist_tiles(p, b) + (p.ks + 127) / 128;
}
__device__ __forceinline__ int sb_q_tiles(const StcaBwdParams& p, int b) { return (sb_targets(p, b) + 127) / 128; }

// Item g -> user b (the last user whose prefix is <= g, which skips users without items) and the
// offset inside that user's items.
__device__ __forceinline__ int sb_find(const int32_t* prefix, int B, int g, int& off) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= g) lo = mid; else hi = mid - 1;
  }
  off = g - prefix[lo];
  return lo;
}

// TMA coordinates of key tile j of (b, h): suffix rows of b, then b's sketch rows.
__device__ __forceinline__ bool sb_key_coord(const StcaBwdParams& p, int b, int h, int j, int D, int& c0, int& row) {
  const int nh = sb_hist_tiles(p, b);
  if (j < nh) {
    c0 = h * D;
    row = p.cu_k[b] + j * 128;
    return false;
  }
  c0 = 0;
  row = (b * p.H + h) * p.ks + (j - nh) * 128;
  return true;
}

__device__ __forceinline__ void sb_drain(SbWaiter& wait, uint64_t* full, int stages, int uses) {
  for (int e = 0; e < stages; ++e) {
    const int fills = (uses > e) ? (uses - e - 1) / stages + 1 : 0;
    if (fills > 0) wait(&full[e], (fills - 1) & 1, true);
  }
}

template <int D>
struct SbLayout {
  static constexpr int KB = D / 64;
  static constexpr int IS = (D == 64) ? 2 : 1;  // item stages
  static constexpr uint32_t tile = KB * kSbBlk;  // [128 rows x D] bf16
  // item operands a, b (K, V or Q, dO); streamed operands c, d (Q, dO or K, V)
  static constexpr uint32_t a_off = 0;
  static constexpr uint32_t b_off = a_off + IS * tile;
  static constexpr uint32_t c_off = b_off + IS * tile;
  static constexpr uint32_t d_off = c_off + 2 * tile;
  static constexpr uint32_t meta_off = d_off + 2 * tile;  // 2 stages x 128 x (lse2, delta, kv length)
  static constexpr uint32_t bar_off = meta_off + 2 * 3 * 128 * 4;
  static constexpr uint32_t total = bar_off + 256;
  static_assert(sizeof(SbBars) <= 256, "barriers");
  static_assert(total <= 227 * 1024, "shared memory");
};

__device__ __forceinline__ void sb_init(SbBars& bars, int is) {
  for (int i = 0; i < is; ++i) {
    mbar_init(&bars.ifull[i], 1);
    mbar_init(&bars.iempty[i], 1);
  }
  for (int i = 0; i < 2; ++i) {
    mbar_init(&bars.sfull2[i], 1);
    mbar_init(&bars.sempty2[i], 1);
  }
  mbar_init(&bars.sfull, 1);
  mbar_init(&bars.pfull, kRowWarps);
  mbar_init(&bars.ofull, 1);
  mbar_init(&bars.ofree, kRowWarps);
  mbar_init(&bars.drain, 1);
  mbar_init(&bars.mready[0], kRowWarps);
  mbar_init(&bars.mready[1], kRowWarps);
  bars.abort_flag = 0;
  fence_mbar_init();
}

// K-major operand of one 16-wide K step s of a [128 rows x D] tile at base
__device__ __forceinline__ uint64_t kdesc(uint32_t base, int s) {
  return sw128_desc(base + (s / 4) * kSbBlk + (s % 4) * 32, 16, 1024);
}
// MN-major B operand (rows = the K index, D contiguous) of K step s (16 rows)
__device__ __forceinline__ uint64_t mndesc(uint32_t base, int s) { return sw128_desc(base + s * 2048, kSbBlk, 1024); }

// A operand (bf16 pairs in TMEM) of K step s over 128 columns packed by column groups: group g holds
// the pairs of columns [kCw g, kCw (g + 1)) in its own TMEM columns [kCw g, kCw g + kCw / 2)
__device__ __forceinline__ uint32_t sb_pairs(uint32_t t, int s) {
  constexpr int kSteps = kCw / 16;  // K steps per group
  return t + (s / kSteps) * kCw + (s % kSteps) * 8;
}

// ===================================================================== key-major: dK, dV
template <int D>
__global__ void __launch_bounds__(kSbThreads, 1)
    stca_bwd_dkv_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapDO,
                        const __grid_constant__ CUtensorMap mapKh, const __grid_constant__ CUtensorMap mapVh,
                        const __grid_constant__ CUtensorMap mapKs, const __grid_constant__ CUtensorMap mapVs,
                        const StcaBwdParams p) {
  using L = SbLayout<D>;
  constexpr int KB = L::KB, IS = L::IS;
  extern __shared__ __align__(1024) uint8_t smem[];
  SbBars& bars = *reinterpret_cast<SbBars*>(smem + L::bar_off);
  if ((smem_u32(smem) & 1023u) != 0) {
    if (threadIdx.x == 0) atomicCAS(&p.hdr->status, 0, (int)SKA_ERR_UNSUPPORTED);
    return;
  }
  uint8_t* sK = smem + L::a_off;
  uint8_t* sV = smem + L::b_off;
  uint8_t* sQ = smem + L::c_off;
  uint8_t* sDO = smem + L::d_off;
  float* sMeta = reinterpret_cast<float*>(smem + L::meta_off);  // stage m: lse2, delta, kv length
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) sb_init(bars, IS);
  if (warp == kProdWarp) {
    tmem_alloc(&bars.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = bars.tmem_base;
  const uint32_t tS = tb, tP = tb + 128, tdV = tb + 256, tdK = tb + 256 + D;
  SbWaiter wait{&bars, &p.hdr->status, p.budget_ns};
  const int nitems = (p.hdr->status == 0) ? p.hdr->total_tiles : 0;

  if (warp == kProdWarp) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      int iuse = 0, suse = 0;
      bool ok = true;
      for (int g = blockIdx.x; g < nitems && ok; g += gridDim.x) {
        int off;
        const int b = sb_find(p.kprefix, p.B, g, off);
        const int nkt = sb_key_tiles(p, b), nqt = sb_q_tiles(p, b);
        const int h = off / nkt, j = off - h * nkt;
        if (nqt == 0) continue;
        const int is = iuse % IS;
        ok = wait(&bars.iempty[is], ((iuse / IS) & 1) ^ 1);
        if (!ok) break;
        int c0, row;
        const bool sk = sb_key_coord(p, b, h, j, D, c0, row);
        mbar_expect_tx(&bars.ifull[is], 2 * L::tile);
        for (int kb = 0; kb < KB; ++kb) {
          tma_load_2d(sK + is * L::tile + kb * kSbBlk, sk ? &mapKs : &mapKh, &bars.ifull[is], c0 + kb * 64, row);
          tma_load_2d(sV + is * L::tile + kb * kSbBlk, sk ? &mapVs : &mapVh, &bars.ifull[is], c0 + kb * 64, row);
        }
        ++iuse;
        for (int qt = 0; qt < nqt && ok; ++qt) {
          const int ss = suse & 1;
          ok = wait(&bars.sempty2[ss], ((suse >> 1) & 1) ^ 1);
          if (!ok) break;
          const int qrow = p.cu_q[b] + qt * 128;
          mbar_expect_tx(&bars.sfull2[ss], 2 * L::tile);
          for (int kb = 0; kb < KB; ++kb) {
            tma_load_2d(sQ + ss * L::tile + kb * kSbBlk, &mapQ, &bars.sfull2[ss], h * D + kb * 64, qrow);
            tma_load_2d(sDO + ss * L::tile + kb * kSbBlk, &mapDO, &bars.sfull2[ss], h * D + kb * 64, qrow);
          }
          ++suse;
        }
      }
      sb_drain(wait, bars.ifull, IS, iuse);
      sb_drain(wait, bars.sfull2, 2, suse);
    }
  } else if (warp == kMmaWarp) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idG = idesc_bf16_f32(128, D, false, true);
      int iuse = 0, suse = 0, npair = 0, nout = 0;
      bool ok = true;
      for (int g = blockIdx.x; g < nitems && ok; g += gridDim.x) {
        int off;
        const int b = sb_find(p.kprefix, p.B, g, off);
        const int nqt = sb_q_tiles(p, b);
        if (nqt == 0) continue;
        const int is = iuse % IS;
        ok = wait(&bars.ifull[is], (iuse / IS) & 1);
        if (!ok) break;
        const uint32_t kbase = smem_u32(sK + is * L::tile), vbase = smem_u32(sV + is * L::tile);
        for (int qt = 0; qt < nqt && ok; ++qt) {
          const int ss = suse & 1;
          ok = wait(&bars.sfull2[ss], (suse >> 1) & 1);
          if (!ok) break;
          const uint32_t qbase = smem_u32(sQ + ss * L::tile), dobase = smem_u32(sDO + ss * L::tile);
          tc_fence_after();
#pragma unroll
          for (int s = 0; s < D / 16; ++s) umma_bf16(tS, kdesc(kbase, s), kdesc(qbase, s), idS, s > 0);
#pragma unroll
          for (int s = 0; s < D / 16; ++s) umma_bf16(tP, kdesc(vbase, s), kdesc(dobase, s), idS, s > 0);
          umma_commit(&bars.sfull);
          ok = wait(&bars.pfull, npair & 1);
          ++npair;
          if (ok && qt == 0 && nout > 0) ok = wait(&bars.ofree, (nout - 1) & 1);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int s = 0; s < 8; ++s) umma_bf16_ts(tdV, sb_pairs(tS, s), mndesc(dobase, s), idG, (qt | s) > 0);
#pragma unroll
          for (int s = 0; s < 8; ++s) umma_bf16_ts(tdK, sb_pairs(tP, s), mndesc(qbase, s), idG, (qt | s) > 0);
          umma_commit(&bars.sempty2[ss]);
          ++suse;
        }
        if (!ok) break;
        umma_commit(&bars.iempty[is]);
        ++iuse;
        umma_commit(&bars.ofull);
        ++nout;
      }
      umma_commit(&bars.drain);
      wait(&bars.drain, 0, true);
    }
  } else {
    // ---------------------------------------------------------------- key rows (warps 0-7)
    const int r = threadIdx.x & 127;     // key row (TMEM lane)
    const int grp = warp >> 2;           // columns [kCw grp, kCw (grp + 1))
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const float c2 = p.scale * kLog2e;
    int npair = 0, nout = 0;
    bool ok = true;
    for (int g = blockIdx.x; g < nitems && ok; g += gridDim.x) {
      int off;
      const int b = sb_find(p.kprefix, p.B, g, off);
      const int nkt = sb_key_tiles(p, b), nqt = sb_q_tiles(p, b), nh = sb_hist_tiles(p, b);
      const int h = off / nkt, j = off - h * nkt;
      const bool sk = j >= nh;
      const int nvalid = sk ? p.ks - (j - nh) * 128 : sb_suffix(p, b) - j * 128;
      const bool keyok = r < nvalid;
      const int kk = j * 128 + r;  // index of this key row in the user's suffix
      float* dv_row = sk ? p.dv_sk + ((static_cast<int64_t>(b) * p.H + h) * p.ks + (j - nh) * 128 + r) * D
                         : p.dv_hist + ((static_cast<int64_t>(p.cu_k[b]) + kk) * p.H + h) * D;
      float* dk_row = sk ? p.dk_sk + ((static_cast<int64_t>(b) * p.H + h) * p.ks + (j - nh) * 128 + r) * D
                         : p.dk_hist + ((static_cast<int64_t>(p.cu_k[b]) + kk) * p.H + h) * D;
      if (nqt == 0) {  // no target reads these keys
        if (keyok && grp == 0)
          for (int c = 0; c < D; c += 4) {
            *reinterpret_cast<float4*>(dv_row + c) = make_float4(0.f, 0.f, 0.f, 0.f);
            *reinterpret_cast<float4*>(dk_row + c) = make_float4(0.f, 0.f, 0.f, 0.f);
          }
        continue;
      }
      const int nt = sb_targets(p, b);
      for (int qt = 0; qt < nqt && ok; ++qt) {
        // The targets of this tile into stage npair & 1: lse (log2 units), delta, and the suffix
        // length they see (-1: no target). A warp writes stage m only after every warp has staged
        // the pair before, hence has finished reading stage m two pairs back.
        const int m = npair & 1;
        float* sLse = sMeta + m * 384;
        float* sDel = sLse + 128;
        int* sKvl = reinterpret_cast<int*>(sLse + 256);
        if (grp == 0) {
          const int tq = qt * 128 + r;
          const int64_t t = static_cast<int64_t>(p.cu_q[b]) + tq;
          const bool tv = tq < nt;
          sLse[r] = tv ? p.lse[t * p.H + h] * kLog2e : 0.f;
          sDel[r] = tv ? p.delta[t * p.H + h] : 0.f;
          sKvl[r] = tv ? (p.kv_len ? max(p.kv_len[t], 0) : INT_MAX) : -1;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.mready[m]);
        ok = __all_sync(0xffffffffu, wait(&bars.mready[m], (npair >> 1) & 1));
        if (!ok) break;
        ok = __all_sync(0xffffffffu, wait(&bars.sfull, npair & 1));
        if (!ok) break;
        ++npair;
        tc_fence_after();
        {
          const int c0 = kCw * grp;
          uint32_t sv[32], dp[32];
          tmem_ld32(tS + lane_off + c0, sv);
          tmem_ld32(tP + lane_off + c0, dp);
          tmem_ld_wait();
          uint32_t pw[16], dw[16];
#pragma unroll
          for (int u = 0; u < 32; u += 4) {
            const float4 ls = *reinterpret_cast<const float4*>(sLse + c0 + u);
            const float4 de = *reinterpret_cast<const float4*>(sDel + c0 + u);
            const int4 kl = *reinterpret_cast<const int4*>(sKvl + c0 + u);
            const float lsv[4] = {ls.x, ls.y, ls.z, ls.w}, dev[4] = {de.x, de.y, de.z, de.w};
            const int klv[4] = {kl.x, kl.y, kl.z, kl.w};
            float pe[4], ds[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const bool v = keyok && (sk ? klv[e] >= 0 : kk < klv[e]);
              pe[e] = v ? ex2_approx(fmaf(__uint_as_float(sv[u + e]), c2, -lsv[e])) : 0.f;
              ds[e] = pe[e] * (__uint_as_float(dp[u + e]) - dev[e]);
            }
            pw[u / 2] = pack_bf16x2(pe[0], pe[1]);
            pw[u / 2 + 1] = pack_bf16x2(pe[2], pe[3]);
            dw[u / 2] = pack_bf16x2(ds[0], ds[1]);
            dw[u / 2 + 1] = pack_bf16x2(ds[2], ds[3]);
          }
          // bf16 pairs over this group's first 16 columns (already read)
          tmem_st16(tS + lane_off + c0, pw);
          tmem_st16(tP + lane_off + c0, dw);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.pfull);
      }
      if (!ok) break;
      ok = __all_sync(0xffffffffu, wait(&bars.ofull, nout & 1));
      if (!ok) break;
      ++nout;
      tc_fence_after();
      {
        // groups 0 .. kGroups/2 - 1 write the dV row, the others the dK row (scaled), D / (kGroups/2)
        // columns each
        constexpr int kCols = D / (kGroups / 2);
        const bool isk = grp >= kGroups / 2;
        const uint32_t src = isk ? tdK : tdV;
        float* dst = isk ? dk_row : dv_row;
        const float mul = isk ? p.scale : 1.f;
        const int cbeg = (grp % (kGroups / 2)) * kCols;
#pragma unroll 1
        for (int c = cbeg; c < cbeg + kCols; c += 32) {
          uint32_t vv[32];
          tmem_ld32(src + lane_off + c, vv);
          tmem_ld_wait();
          if (keyok) {
#pragma unroll
            for (int u = 0; u < 32; u += 4)
              *reinterpret_cast<float4*>(dst + c + u) =
                  make_float4(mul * __uint_as_float(vv[u]), mul * __uint_as_float(vv[u + 1]),
                              mul * __uint_as_float(vv[u + 2]), mul * __uint_as_float(vv[u + 3]));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.ofree);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kProdWarp) {
    tc_fence_after();
    tmem_dealloc(tb, 512);
  }
}

// ===================================================================== query-major: dq
template <int D>
__global__ void __launch_bounds__(kSbThreads, 1)
    stca_bwd_dq_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapDO,
                       const __grid_constant__ CUtensorMap mapKh, const __grid_constant__ CUtensorMap mapVh,
                       const __grid_constant__ CUtensorMap mapKs, const __grid_constant__ CUtensorMap mapVs,
                       const StcaBwdParams p) {
  using L = SbLayout<D>;
  constexpr int KB = L::KB, IS = L::IS;
  extern __shared__ __align__(1024) uint8_t smem[];
  SbBars& bars = *reinterpret_cast<SbBars*>(smem + L::bar_off);
  if ((smem_u32(smem) & 1023u) != 0) {
    if (threadIdx.x == 0) atomicCAS(&p.hdr->status, 0, (int)SKA_ERR_UNSUPPORTED);
    return;
  }
  uint8_t* sQ = smem + L::a_off;
  uint8_t* sDO = smem + L::b_off;
  uint8_t* sK = smem + L::c_off;
  uint8_t* sV = smem + L::d_off;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) sb_init(bars, IS);
  if (warp == kProdWarp) {
    tmem_alloc(&bars.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = bars.tmem_base;
  const uint32_t tS = tb, tP = tb + 128, tdQ = tb + 256;
  SbWaiter wait{&bars, &p.hdr->status, p.budget_ns};
  const int nitems = (p.hdr->status == 0) ? p.hdr->tiles_per_cluster : 0;

  if (warp == kProdWarp) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      int iuse = 0, suse = 0;
      bool ok = true;
      for (int g = blockIdx.x; g < nitems && ok; g += gridDim.x) {
        int off;
        const int b = sb_find(p.qprefix, p.B, g, off);
        const int nkt = sb_key_tiles(p, b), nqt = sb_q_tiles(p, b);
        const int h = off / nqt, qt = off - h * nqt;
        if (nkt == 0) continue;
        const int is = iuse % IS;
        ok = wait(&bars.iempty[is], ((iuse / IS) & 1) ^ 1);
        if (!ok) break;
        const int qrow = p.cu_q[b] + qt * 128;
        mbar_expect_tx(&bars.ifull[is], 2 * L::tile);
        for (int kb = 0; kb < KB; ++kb) {
          tma_load_2d(sQ + is * L::tile + kb * kSbBlk, &mapQ, &bars.ifull[is], h * D + kb * 64, qrow);
          tma_load_2d(sDO + is * L::tile + kb * kSbBlk, &mapDO, &bars.ifull[is], h * D + kb * 64, qrow);
        }
        ++iuse;
        for (int j = 0; j < nkt && ok; ++j) {
          const int ss = suse & 1;
          ok = wait(&bars.sempty2[ss], ((suse >> 1) & 1) ^ 1);
          if (!ok) break;
          int c0, row;
          const bool sk = sb_key_coord(p, b, h, j, D, c0, row);
          mbar_expect_tx(&bars.sfull2[ss], 2 * L::tile);
          for (int kb = 0; kb < KB; ++kb) {
            tma_load_2d(sK + ss * L::tile + kb * kSbBlk, sk ? &mapKs : &mapKh, &bars.sfull2[ss], c0 + kb * 64, row);
            tma_load_2d(sV + ss * L::tile + kb * kSbBlk, sk ? &mapVs : &mapVh, &bars.sfull2[ss], c0 + kb * 64, row);
          }
          ++suse;
        }
      }
      sb_drain(wait, bars.ifull, IS, iuse);
      sb_drain(wait, bars.sfull2, 2, suse);
    }
  } else if (warp == kMmaWarp) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idG = idesc_bf16_f32(128, D, false, true);
      int iuse = 0, suse = 0, npair = 0, nchain = 0;
      bool ok = true;
      for (int g = blockIdx.x; g < nitems && ok; g += gridDim.x) {
        int off;
        const int b = sb_find(p.qprefix, p.B, g, off);
        const int nkt = sb_key_tiles(p, b);
        if (nkt == 0) continue;
        const int is = iuse % IS;
        ok = wait(&bars.ifull[is], (iuse / IS) & 1);
        if (!ok) break;
        const uint32_t qbase = smem_u32(sQ + is * L::tile), dobase = smem_u32(sDO + is * L::tile);
        for (int j = 0; j < nkt && ok; ++j) {
          const int ss = suse & 1;
          ok = wait(&bars.sfull2[ss], (suse >> 1) & 1);
          if (!ok) break;
          const uint32_t kbase = smem_u32(sK + ss * L::tile), vbase = smem_u32(sV + ss * L::tile);
          tc_fence_after();
#pragma unroll
          for (int s = 0; s < D / 16; ++s) umma_bf16(tS, kdesc(qbase, s), kdesc(kbase, s), idS, s > 0);
#pragma unroll
          for (int s = 0; s < D / 16; ++s) umma_bf16(tP, kdesc(dobase, s), kdesc(vbase, s), idS, s > 0);
          umma_commit(&bars.sfull);
          ok = wait(&bars.pfull, npair & 1);
          ++npair;
          const int cj = j % kDqChain;
          if (ok && cj == 0 && nchain > 0) ok = wait(&bars.ofree, (nchain - 1) & 1);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int s = 0; s < 8; ++s) umma_bf16_ts(tdQ, sb_pairs(tS, s), mndesc(kbase, s), idG, (cj | s) > 0);
#pragma unroll
          for (int s = 0; s < 8; ++s) umma_bf16_ts(tdQ, sb_pairs(tP, s), mndesc(kbase, s), idG, 1u);
          umma_commit(&bars.sempty2[ss]);
          ++suse;
          if (cj == kDqChain - 1 || j == nkt - 1) {
            umma_commit(&bars.ofull);
            ++nchain;
          }
        }
        if (!ok) break;
        umma_commit(&bars.iempty[is]);
        ++iuse;
      }
      umma_commit(&bars.drain);
      wait(&bars.drain, 0, true);
    }
  } else {
    // ---------------------------------------------------------------- target rows (warps 0-7)
    const int r = threadIdx.x & 127;     // target row (TMEM lane)
    const int grp = warp >> 2;           // key columns [kCw grp, kCw (grp + 1)), dq columns [D/kGroups grp, ...)
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const float c2 = p.scale * kLog2e;
    int npair = 0, nchain = 0;
    bool ok = true;
    for (int g = blockIdx.x; g < nitems && ok; g += gridDim.x) {
      int off;
      const int b = sb_find(p.qprefix, p.B, g, off);
      const int nkt = sb_key_tiles(p, b), nqt = sb_q_tiles(p, b), nh = sb_hist_tiles(p, b);
      const int h = off / nqt, qt = off - h * nqt;
      const int tq = qt * 128 + r;
      const bool tv = tq < sb_targets(p, b);
      const int64_t t = static_cast<int64_t>(p.cu_q[b]) + tq;
      float* dq_row = p.dq + (t * p.H + h) * D;
      if (nkt == 0) {  // no keys: the output is zero
        if (tv && grp == 0)
          for (int c = 0; c < D; c += 4) *reinterpret_cast<float4*>(dq_row + c) = make_float4(0.f, 0.f, 0.f, 0.f);
        continue;
      }
      const float lse2 = tv ? p.lse[t * p.H + h] * kLog2e : 0.f;
      const float del = tv ? p.delta[t * p.H + h] : 0.f;
      int hl = sb_suffix(p, b);
      if (p.kv_len && tv) hl = min(hl, max(p.kv_len[t], 0));
      for (int j = 0; j < nkt && ok; ++j) {
        const int nvalid = !tv ? 0 : (j < nh ? hl - j * 128 : p.ks - (j - nh) * 128);
        ok = __all_sync(0xffffffffu, wait(&bars.sfull, npair & 1));
        if (!ok) break;
        ++npair;
        tc_fence_after();
        {
          const int c0 = kCw * grp;
          uint32_t sv[32], dp[32];
          tmem_ld32(tS + lane_off + c0, sv);
          tmem_ld32(tP + lane_off + c0, dp);
          tmem_ld_wait();
          uint32_t hw[16], lw[16];
          const uint64_t del2 = f2_pack(del, del);
#pragma unroll
          for (int u = 0; u < 32; u += 2) {
            float pe[2];
#pragma unroll
            for (int e = 0; e < 2; ++e)
              pe[e] = (c0 + u + e < nvalid) ? ex2_approx(fmaf(__uint_as_float(sv[u + e]), c2, -lse2)) : 0.f;
            const uint64_t ds = f2_mul(f2_pack(pe[0], pe[1]),
                                       f2_sub(f2_pack(__uint_as_float(dp[u]), __uint_as_float(dp[u + 1])), del2));
            split_bf16x2(ds, hw[u / 2], lw[u / 2]);
          }
          // hi over S, lo over dP: this group's first 16 columns of each (already read)
          tmem_st16(tS + lane_off + c0, hw);
          tmem_st16(tP + lane_off + c0, lw);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.pfull);
        if (j % kDqChain == kDqChain - 1 || j == nkt - 1) {
          // end of a chain: add it into the output row (the first chain writes it)
          ok = __all_sync(0xffffffffu, wait(&bars.ofull, nchain & 1));
          if (!ok) break;
          ++nchain;
          tc_fence_after();
          const bool first = j < kDqChain;
#pragma unroll 1
          for (int c = grp * (D / kGroups); c < (grp + 1) * (D / kGroups); c += 16) {
            uint32_t qv[16];
            tmem_ld16(tdQ + lane_off + c, qv);
            tmem_ld_wait();
            if (tv) {
#pragma unroll
              for (int u = 0; u < 16; u += 4) {
                float4 a = make_float4(p.scale * __uint_as_float(qv[u]), p.scale * __uint_as_float(qv[u + 1]),
                                       p.scale * __uint_as_float(qv[u + 2]), p.scale * __uint_as_float(qv[u + 3]));
                if (!first) {
                  const float4 o = *reinterpret_cast<const float4*>(dq_row + c + u);
                  a.x += o.x;
                  a.y += o.y;
                  a.z += o.z;
                  a.w += o.w;
                }
                *reinterpret_cast<float4*>(dq_row + c + u) = a;
              }
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars.ofree);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kProdWarp) {
    tc_fence_after();
    tmem_dealloc(tb, 512);
  }
}

// ===================================================================== small kernels
// Per-user item prefixes (key tiles x heads, query tiles x heads) and their totals; clears the
// status word. One thread: the users are walked once.
__global__ void stca_bwd_schedule_kernel(StcaBwdParams p) {
  if (blockIdx.x != 0 || threadIdx.x != 0) return;
  int64_t kt = 0, qt = 0;
  p.kprefix[0] = 0;
  p.qprefix[0] = 0;
  for (int b = 0; b < p.B; ++b) {
    kt += static_cast<int64_t>(p.H) * sb_key_tiles(p, b);
    qt += static_cast<int64_t>(p.H) * sb_q_tiles(p, b);
    p.kprefix[b + 1] = static_cast<int32_t>(min(kt, int64_t(INT_MAX)));
    p.qprefix[b + 1] = static_cast<int32_t>(min(qt, int64_t(INT_MAX)));
  }
  const bool too_many = kt >= INT_MAX || qt >= INT_MAX;
  p.hdr->total_tiles = too_many ? 0 : static_cast<int32_t>(kt);
  p.hdr->tiles_per_cluster = too_many ? 0 : static_cast<int32_t>(qt);
  p.hdr->status = too_many ? static_cast<int>(SKA_ERR_INVALID_VALUE) : 0;
}

// delta[t, h] = <dO[t, h, :], out[t, h, :]>, one warp per row.
__global__ void stca_bwd_delta_kernel(const __nv_bfloat16* dout, const float* out, float* delta, int64_t rows, int D) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); row < rows;
       row += warps) {
    float s = 0.f;
    for (int c = lane; c < D; c += 32) s = fmaf(__bfloat162float(dout[row * D + c]), out[row * D + c], s);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) delta[row] = s;
  }
}

// After a device-side error, every gradient of the call becomes NaN.
__global__ void stca_bwd_poison_kernel(const int* status, float* a, int64_t na, float* b, int64_t nb, float* c,
                                       int64_t nc, float* d, int64_t nd, float* e, int64_t ne) {
  if (*reinterpret_cast<const volatile int*>(status) == 0) return;
  const float nan = __int_as_float(0x7fc00000);
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t i0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  for (int64_t i = i0; i < na; i += stride) a[i] = nan;
  for (int64_t i = i0; i < nb; i += stride) b[i] = nan;
  for (int64_t i = i0; i < nc; i += stride) c[i] = nan;
  for (int64_t i = i0; i < nd; i += stride) d[i] = nan;
  for (int64_t i = i0; i < ne; i += stride) e[i] = nan;
}

template <int D>
cudaError_t stca_bwd_launch_t(int ctas_kv, int ctas_q, const CUtensorMap* maps, const StcaBwdParams& p,
                              cudaStream_t s) {
  const size_t smem = SbLayout<D>::total;
  auto k1 = stca_bwd_dkv_kernel<D>;
  auto k2 = stca_bwd_dq_kernel<D>;
  cudaError_t e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  if (ctas_kv > 0) k1<<<ctas_kv, kSbThreads, smem, s>>>(maps[0], maps[1], maps[2], maps[3], maps[4], maps[5], p);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (ctas_q > 0) k2<<<ctas_q, kSbThreads, smem, s>>>(maps[0], maps[1], maps[2], maps[3], maps[4], maps[5], p);
  return cudaGetLastError();
}

}  // namespace

bool stca_bwd_supported(int D) { return D == 64 || D == 128; }

cudaError_t launch_stca_bwd_prep(const StcaBwdParams& p, const void* dout, const float* out, int64_t rows, int D,
                                 cudaStream_t s) {
  stca_bwd_schedule_kernel<<<1, 32, 0, s>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || rows == 0) return e;
  const int blocks = static_cast<int>(std::min<int64_t>((rows + 7) / 8, 148 * 8));
  stca_bwd_delta_kernel<<<blocks, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(dout), out, p.delta, rows, D);
  return cudaGetLastError();
}

cudaError_t launch_stca_bwd(int D, int ctas_kv, int ctas_q, const CUtensorMap* maps, const StcaBwdParams& p,
                            cudaStream_t s) {
  if (D == 64) return stca_bwd_launch_t<64>(ctas_kv, ctas_q, maps, p, s);
  if (D == 128) return stca_bwd_launch_t<128>(ctas_kv, ctas_q, maps, p, s);
  return cudaErrorInvalidValue;
}

cudaError_t launch_stca_bwd_poison(const StcaBwdParams& p, int64_t nq, int64_t nh, int64_t ns, cudaStream_t s) {
  stca_bwd_poison_kernel<<<2 * 148, 256, 0, s>>>(&p.hdr->status, p.dq, nq, p.dk_hist, nh, p.dv_hist, nh, p.dk_sk, ns,
                                                 p.dv_sk, ns);
  return cudaGetLastError();
}

}  // namespace ska
