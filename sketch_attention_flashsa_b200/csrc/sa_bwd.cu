// SA backward on sm_100a: gradients of <dSketch, sketch> through SequenceO1 §3.1 Eq. (7)-(9)
// (SA is trained end to end, App. A.4), for both normalisations.
//
// Per 128-token tile of one (user, head), one CTA holding the launch's KP <= 256 prototypes, tokens on
// TMEM lanes (S^T orientation):
//   MMA  S^T  = K . Q^T                        -> A = exp(scale s - lse) (PROTO: per-token lse;
//                                                 TOKEN: per-prototype lse), to smem in bf16
//   MMA  dV   = A^T . dO        (M=tok, N=d)   -> TMEM (A as hi + lo over prototype chunks)
//   MMA  dA^T = V . dO^T        (M=tok, N=k)   -> TMEM (over S^T)
//   softmax-gradient: PROTO dS = A (dA - delta_i) with delta_i = sum_j A_ji dA_ji in fp32 (each
//        warpgroup sums its half of the prototypes, the halves are added in a fixed order);
//        TOKEN dS = A (dA - D_j) with D_j = dO_j . O_j from the forward sketch. dS goes to smem
//        as a bf16 pair hi + lo (16 significant bits).
//   MMA  dK   = dS^T . Q        (M=tok, N=d)   -> TMEM from the hi half (both halves over prototype
//        chunks), scaled on the way out
//   MMA  dQ  += dS . K          (M=proto, N=d) -> TMEM, both halves; restarted every 16 tiles and
//        added into the CTA's partial slot (the tensor core's fp32 accumulation is not
//        round-to-nearest, so one chain over a whole segment would drift); a second kernel sums
//        the partial slots of every prototype set in a fixed order.
// Warps 0-7 (two warpgroups, each owning half of the prototype columns) do the elementwise
// work; thread 0 also issues the TMA loads and MMAs. The phases of a tile run one after another.
//
// Prototype sets larger than one CTA holds (TMEM: S^T, dV, dK and the dQ blocks) run as one
// launch per chunk of KP prototypes (rows j0 .. j0 + KP - 1 of Q, dO, the sketch and TOKEN's lse):
// every chunk but the first adds its dK and dV to the previous chunk's, and the chunk's dQ slots
// are reduced into dq's rows j0 ... PROTO's delta_i sums over all k prototypes of the token, so
// a first pass per chunk (pass 1: S, A and dA^T only) adds its part into a [T, H] buffer in chunk
// order, and the gradient pass (pass 2) reads delta_i from there.
#include <algorithm>
#include <cmath>

#include "ska_internal.h"
#include "ska_ptx.cuh"

namespace ska {

namespace {

constexpr int kBwdThreads = 256;
constexpr int kBwdWarps = 8;
constexpr int kBlk = 16384;  // [128 rows x 64 bf16] swizzled block
constexpr int kDqFlush = 16;  // tiles per dQ accumulation chain in TMEM
// Larger prototype sets run as launches over chunks of prototypes (see sa_bwd_chunk).
constexpr int kMaxChunkedProtos = 4096;

struct BwdLayout {
  uint32_t q_off, do_off, k_off, v_off, a_off, lo_off, lse_off, d_off, bar_off, total;
};

// Q, dO: ceil(d/64) blocks of k rows x 128 B (k padded to a multiple of 8);
// K, V: d/64 blocks of 128 rows; A / dS_hi and dS_lo: ceil(k/64) blocks of 128 rows.
__host__ __device__ inline BwdLayout bwd_layout(int D, int k) {
  BwdLayout L;
  const uint32_t kb = D / 64, pb = (k + 63) / 64;
  const uint32_t qbytes = kb * ((k * 128 + 1023) & ~1023u);
  uint32_t off = 0;
  L.q_off = off;
  off += qbytes;
  L.do_off = off;
  off += qbytes;
  L.k_off = off;
  off += kb * kBlk;
  L.v_off = off;
  off += kb * kBlk;
  L.a_off = off;
  off += max(pb, 2u) * kBlk;  // MMA for dQ reads a full 128-prototype block
  L.lo_off = off;
  off += max(pb, 2u) * kBlk;
  L.lse_off = off;
  off += 256 * 4;
  L.d_off = off;
  off += 256 * 4;
  L.bar_off = off;
  off += 128;  // mbarriers, TMEM base, abort flag
  L.total = off;
  return L;
}

__host__ __device__ inline int bwd_tmem_cols(int D, int k) { return k + 2 * D + ((k + 127) / 128) * D; }

struct BwdBars {
  uint64_t ldk, ldv, qd, m1, a, m2, ds, m3, drain, dready, dl;
  uint32_t tmem_base;
  int abort_flag;
};

static_assert(sizeof(BwdBars) <= 128, "barrier area");

struct BwdPos {
  int b, h, j, nb;
};

__device__ __forceinline__ int bwd_used(const SaBwdParams& p, int b) {
  int len = p.cu_seqlens[b + 1] - p.cu_seqlens[b];
  if (p.seqused) len = min(len, p.seqused[b]);
  return max(len, 0);
}

__device__ __forceinline__ void bwd_seek(const SaBwdParams& p, int g, BwdPos& t) {
  int lo = 0, hi = p.B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.H * p.tile_prefix[mid] <= g) lo = mid; else hi = mid - 1;
  }
  t.b = lo;
  t.nb = p.tile_prefix[lo + 1] - p.tile_prefix[lo];
  const int off = g - p.H * p.tile_prefix[lo];
  t.h = off / t.nb;
  t.j = off - t.h * t.nb;
}

__device__ __forceinline__ void bwd_next(const SaBwdParams& p, BwdPos& t) {
  if (++t.j < t.nb) return;
  t.j = 0;
  if (++t.h < p.H) return;
  t.h = 0;
  do {
    ++t.b;
    if (t.b >= p.B) return;
    t.nb = p.tile_prefix[t.b + 1] - p.tile_prefix[t.b];
  } while (t.nb == 0);
}

struct BwdWaiter {
  BwdBars* bars;
  int* status;
  uint64_t budget;
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


// CHUNK: this launch is one chunk of a larger prototype set (passes 1 and 2, dK/dV accumulation);
// without it those paths are compiled out.
template <int D, int KP, bool CHUNK>
__global__ void __launch_bounds__(kBwdThreads, 1)
    sa_bwd_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapDO,
                  const __grid_constant__ CUtensorMap mapK, const __grid_constant__ CUtensorMap mapV,
                  const SaBwdParams p, const __grid_constant__ SaBwdChunk ck) {
  constexpr int KB = D / 64;
  constexpr int NCOL = KP / 2;                  // prototype columns per worker thread
  constexpr int QBLK = (KP * 128 + 1023) & ~1023;
  constexpr int CV = (KP + 31) / 32 * 32;      // TMEM columns: S^T/dA^T at 0, dV, dK, dQ blocks
  constexpr int CK = CV + D;
  constexpr int CQ = CK + D;
  constexpr int QBLOCKS = (KP + 127) / 128;
  static_assert(CQ + QBLOCKS * D <= 512, "TMEM");
  static_assert(NCOL % 8 == 0, "columns");
  // No static shared memory: the dynamic region starts on a 1024-byte boundary (checked below)
  // and holds the barriers too, so that k = 256, d = 64 fits without alignment slack.
  extern __shared__ __align__(1024) uint8_t smem[];
  const BwdLayout L = bwd_layout(D, KP);
  BwdBars& bars = *reinterpret_cast<BwdBars*>(smem + L.bar_off);
  uint64_t& dready = bars.dready;
  if ((smem_u32(smem) & 1023u) != 0) {
    if (threadIdx.x == 0) atomicCAS(&p.hdr->status, 0, (int)SKA_ERR_UNSUPPORTED);
    return;
  }
  uint8_t* sQ = smem + L.q_off;
  uint8_t* sDO = smem + L.do_off;
  uint8_t* sK = smem + L.k_off;
  uint8_t* sV = smem + L.v_off;
  uint8_t* sA = smem + L.a_off;    // A hi, then dS hi
  uint8_t* sLo = smem + L.lo_off;  // A lo, then dS lo
  float* sLse = reinterpret_cast<float*>(smem + L.lse_off);
  float* sDl = sLse;  // PROTO (no per-prototype lse): each warpgroup's partial delta per token
  float* sDj = reinterpret_cast<float*>(smem + L.d_off);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(&bars.ldk, 1);
    mbar_init(&bars.ldv, 1);
    mbar_init(&bars.qd, 1);
    mbar_init(&bars.m1, 1);
    mbar_init(&bars.m2, 1);
    mbar_init(&bars.m3, 1);
    mbar_init(&bars.a, kBwdWarps);
    mbar_init(&bars.ds, kBwdWarps);
    mbar_init(&dready, kBwdWarps);
    mbar_init(&bars.dl, kBwdWarps);
    mbar_init(&bars.drain, 1);
    bars.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&bars.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = bars.tmem_base;
  BwdWaiter wait{&bars, &p.hdr->status, p.budget_ns};
  const int total = p.hdr->total_tiles;
  const int W = p.hdr->tiles_per_cluster;
  const int g0 = blockIdx.x * W;
  const int ntiles = (W > 0 && g0 < total) ? (min(total, g0 + W) - g0) : 0;

  // One program for all 256 threads; thread 0 also issues the TMA loads and the MMAs of each
  // phase (the phases of a tile are sequential, so no separate control warp is needed).
  constexpr uint32_t i1 = idesc_bf16_f32(128, KP, false, false);
  constexpr uint32_t iV = idesc_bf16_f32(128, D, false, true);
  constexpr uint32_t iQ = idesc_bf16_f32(128, D, true, true);
  const bool ctl = (threadIdx.x == 0);
  const int pass = CHUNK ? ck.pass : 0;
  const bool accumulate = CHUNK && ck.accumulate;
  const int wg = warp >> 2, q4 = warp & 3;
  const int r = q4 * 32 + lane;
  const int col0 = wg * NCOL;
  const uint32_t loff = static_cast<uint32_t>(q4 * 32) << 16;
  const float L2E = 1.4426950408889634f;
  const float c2 = p.scale * L2E;
  int nk_issued = 0, nv_issued = 0, nq_issued = 0;  // fills requested (thread 0)
  int nk_seen = 0, nv_seen = 0;                        // fills waited for
  auto load_qdo = [&](const BwdPos& u) {
    ++nq_issued;
    const int qrow = (p.q_per_user ? u.b * p.H * ck.kt : 0) + u.h * ck.kt + ck.j0;
    const int orow = (u.b * p.H + u.h) * ck.kt + ck.j0;
    mbar_expect_tx(&bars.qd, 2 * KB * KP * 128);
    for (int kb = 0; kb < KB; ++kb) {
      tma_load_2d(sQ + kb * QBLK, &mapQ, &bars.qd, kb * 64, qrow);
      tma_load_2d(sDO + kb * QBLK, &mapDO, &bars.qd, kb * 64, orow);
    }
  };
  auto load_k = [&](const BwdPos& u) {
    ++nk_issued;
    const int row = p.cu_seqlens[u.b] + u.j * 128;
    mbar_expect_tx(&bars.ldk, KB * kBlk);
    for (int kb = 0; kb < KB; ++kb) tma_load_2d(sK + kb * kBlk, &mapK, &bars.ldk, u.h * D + kb * 64, row);
  };
  auto load_v = [&](const BwdPos& u) {
    ++nv_issued;
    const int row = p.cu_seqlens[u.b] + u.j * 128;
    mbar_expect_tx(&bars.ldv, KB * kBlk);
    for (int kb = 0; kb < KB; ++kb) tma_load_2d(sV + kb * kBlk, &mapV, &bars.ldv, u.h * D + kb * 64, row);
  };
  BwdPos t;
  if (ntiles > 0) bwd_seek(p, g0, t);
  int nseg = 0;
  int segt = 0;  // tile index inside this CTA's part of the current (user, head) segment
  bool ok = true;
  for (int i = 0; i < ntiles && ok; ++i) {
    const bool first = (t.j == 0) || (i == 0);
    const bool last = (t.j == t.nb - 1) || (i == ntiles - 1);
    segt = first ? 0 : segt + 1;
    // dQ restarts in TMEM every kDqFlush tiles and is added into the partial slot: the tensor
    // core's fp32 accumulation is not round-to-nearest, so long chains would drift
    const bool fresh = (segt % kDqFlush) == 0;
    const bool flush = last || (segt % kDqFlush) == kDqFlush - 1;
    const int used = bwd_used(p, t.b);
    const int tok0 = p.cu_seqlens[t.b] + t.j * 128;
    const int tok = tok0 + r;
    const bool valid = (t.j * 128 + r) < used;
    // this row's lse, requested before the waits (PROTO)
    const float lrow = (p.norm == SKA_NORM_PROTO && valid) ? p.lse[static_cast<int64_t>(tok) * p.H + t.h] * L2E : 0.f;
    if (ctl && i == 0) {  // later tiles' loads are issued as soon as the previous tile frees the buffers
      load_qdo(t);
      load_v(t);
      load_k(t);
    }
    if (ctl && i + 2 < ntiles) {  // K and V two tiles ahead into L2
      BwdPos t2 = t;
      bwd_next(p, t2);
      bwd_next(p, t2);
      const int row = p.cu_seqlens[t2.b] + t2.j * 128;
      for (int kb = 0; kb < KB; ++kb) {
        tma_prefetch_l2_2d(&mapK, t2.h * D + kb * 64, row);
        tma_prefetch_l2_2d(&mapV, t2.h * D + kb * 64, row);
      }
    }
    if (first && p.norm == SKA_NORM_TOKEN) {
      // per-prototype lse (log2 units) and D_j = dO_j . O_j of this (user, head)
      const int jj = threadIdx.x;
      if (jj < p.k) {
        const int64_t row = (static_cast<int64_t>(t.b) * p.H + t.h) * ck.kt + ck.j0 + jj;
        sLse[jj] = p.lse[row] * L2E;
        float acc = 0.f;
        for (int dd = 0; dd < D; ++dd) acc += __bfloat162float(p.dsketch[row * D + dd]) * p.sketch[row * D + dd];
        sDj[jj] = acc;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&dready);
      ok = __all_sync(0xffffffffu, wait(&dready, nseg & 1));
      if (!ok) break;
    }
    ok = __all_sync(0xffffffffu, wait(&bars.ldk, i & 1) && wait(&bars.ldv, i & 1) &&
                                     (!first || wait(&bars.qd, nseg & 1)));
    nk_seen = nv_seen = i + 1;
    if (!ok) break;
    if (ctl) {
      tc_fence_after();
#pragma unroll
      for (int s = 0; s < D / 16; ++s)
        umma_bf16(tb, sw128_desc(smem_u32(sK) + (s / 4) * kBlk + (s % 4) * 32, 16, 1024),
                  sw128_desc(smem_u32(sQ) + (s / 4) * QBLK + (s % 4) * 32, 16, 1024), i1, s > 0);
      umma_commit(&bars.m1);
    }
    ok = __all_sync(0xffffffffu, wait(&bars.m1, i & 1));
    if (!ok) break;
    tc_fence_after();
    // A = exp(scale s - lse): PROTO per token row, TOKEN per prototype column
    float a[NCOL];
    {
      uint32_t sv[NCOL];
#pragma unroll
      for (int c = 0; c < NCOL; c += 8) tmem_ld8(tb + loff + col0 + c, sv + c);
      tmem_ld_wait();
#pragma unroll
      for (int c = 0; c < NCOL; ++c) {
        const float l2 = (p.norm == SKA_NORM_PROTO) ? lrow : sLse[col0 + c];
        a[c] = valid ? ex2_approx(__uint_as_float(sv[c]) * c2 - l2) : 0.f;
      }
    }
    // A in bf16 for dV = A^T dO (fp32 A stays in registers for dS): dV_i is a weighted mean of
    // dO rows, so rounding the weights to 8 significant bits leaves ~1e-3 relative error in dV
    // (over chunks of a larger prototype set, dV sums more prototypes and grows with them: A then
    // enters as a bf16 pair hi + lo)
    if (pass != 1) {
#pragma unroll
      for (int c = 0; c < NCOL; c += 8) {
        const int jj = col0 + c;
        const uint32_t off = (jj >> 6) * kBlk + sw128_offset(r, (jj & 63) * 2);
        if constexpr (CHUNK) {
          uint32_t wh[4], wl[4];
#pragma unroll
          for (int u = 0; u < 8; u += 2) split_bf16x2(f2_pack(a[c + u], a[c + u + 1]), wh[u / 2], wl[u / 2]);
          *reinterpret_cast<uint4*>(sA + off) = make_uint4(wh[0], wh[1], wh[2], wh[3]);
          *reinterpret_cast<uint4*>(sLo + off) = make_uint4(wl[0], wl[1], wl[2], wl[3]);
        } else {
          *reinterpret_cast<uint4*>(sA + off) = make_uint4(pack_bf16x2(a[c], a[c + 1]), pack_bf16x2(a[c + 2], a[c + 3]),
                                                           pack_bf16x2(a[c + 4], a[c + 5]), pack_bf16x2(a[c + 6], a[c + 7]));
        }
      }
    }
    fence_async_shared();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars.a);
    if (ctl) {
      ok = wait(&bars.a, i & 1);
      if (ok) {
        tc_fence_after();
        if (pass != 1) {
#pragma unroll
          for (int s = 0; s < KP / 16; ++s)
            umma_bf16(tb + CV, sw128_desc(smem_u32(sA) + (s / 4) * kBlk + (s % 4) * 32, 16, 1024),
                      sw128_desc(smem_u32(sDO) + s * 2048, QBLK, 1024), iV, s > 0);
          if constexpr (CHUNK) {
#pragma unroll
            for (int s = 0; s < KP / 16; ++s)
              umma_bf16(tb + CV, sw128_desc(smem_u32(sLo) + (s / 4) * kBlk + (s % 4) * 32, 16, 1024),
                        sw128_desc(smem_u32(sDO) + s * 2048, QBLK, 1024), iV, 1u);
          }
        }
#pragma unroll
        for (int s = 0; s < D / 16; ++s)
          umma_bf16(tb, sw128_desc(smem_u32(sV) + (s / 4) * kBlk + (s % 4) * 32, 16, 1024),
                    sw128_desc(smem_u32(sDO) + (s / 4) * QBLK + (s % 4) * 32, 16, 1024), i1, s > 0);
        umma_commit(&bars.m2);
      }
    }
    ok = __all_sync(0xffffffffu, wait(&bars.m2, i & 1));
    if (!ok) break;
    tc_fence_after();
    BwdPos tn = t;  // the next tile of this CTA
    if (i + 1 < ntiles) bwd_next(p, tn);
    if (ctl && i + 1 < ntiles) load_v(tn);  // the MMAs reading V are complete
    // PROTO: delta_i = sum_j A_ij dA_ij in fp32; each warpgroup sums its half of the
    // prototypes and the two halves are added in a fixed order
    float delta = 0.f;
    if (p.norm == SKA_NORM_PROTO && pass == 2) {
      delta = (valid && tok < p.total_tokens) ? ck.delta[static_cast<int64_t>(tok) * p.H + t.h] : 0.f;
    } else if (p.norm == SKA_NORM_PROTO) {
      float part = 0.f;
#pragma unroll
      for (int c = 0; c < NCOL; c += 16) {
        uint32_t da[16];
        if constexpr (NCOL >= 16) {
          tmem_ld16(tb + loff + col0 + c, da);
        } else {
          tmem_ld8(tb + loff + col0 + c, da);
        }
        tmem_ld_wait();
#pragma unroll
        for (int u = 0; u < (NCOL >= 16 ? 16 : 8); ++u) part = fmaf(a[c + u], __uint_as_float(da[u]), part);
      }
      sDl[wg * 128 + r] = part;
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.dl);
      ok = __all_sync(0xffffffffu, wait(&bars.dl, i & 1));
      if (!ok) break;
      delta = sDl[r] + sDl[128 + r];
    }
    if (pass == 1) {
      // this chunk's part of delta_i, added in chunk order (launches run one after another)
      if (wg == 0 && valid && tok < p.total_tokens) {
        float* dp = ck.delta + static_cast<int64_t>(tok) * p.H + t.h;
        *dp = (ck.j0 == 0 ? 0.f : *dp) + delta;
      }
      tc_fence_before();
      __syncwarp();
      if (ctl && i + 1 < ntiles) {  // the MMAs of this tile are complete: K, Q and dO are free
        if (tn.j == 0) load_qdo(tn);
        load_k(tn);
      }
      if (first) ++nseg;
      t = tn;
      continue;
    }
    // dS = A (dA - delta) as a bf16 pair hi + lo
    constexpr int DC = (NCOL >= 16) ? 16 : 8;  // columns per TMEM round trip
#pragma unroll
    for (int c0 = 0; c0 < NCOL; c0 += DC) {
      uint32_t da[DC];
      if constexpr (DC == 16) {
        tmem_ld16(tb + loff + col0 + c0, da);
      } else {
        tmem_ld8(tb + loff + col0 + c0, da);
      }
      tmem_ld_wait();
#pragma unroll
      for (int h8 = 0; h8 < DC; h8 += 8) {
        const int c = c0 + h8;
        uint32_t wh[4], wl[4];
#pragma unroll
        for (int u = 0; u < 8; u += 2) {  // in fp32 pairs
          const uint64_t sub = (p.norm == SKA_NORM_PROTO) ? f2_pack(delta, delta)
                                                          : f2_pack(sDj[col0 + c + u], sDj[col0 + c + u + 1]);
          const uint64_t ds = f2_mul(f2_pack(a[c + u], a[c + u + 1]),
                                     f2_sub(f2_pack(__uint_as_float(da[h8 + u]), __uint_as_float(da[h8 + u + 1])), sub));
          split_bf16x2(ds, wh[u / 2], wl[u / 2]);
        }
        const int jj = col0 + c;
        const uint32_t off = (jj >> 6) * kBlk + sw128_offset(r, (jj & 63) * 2);
        *reinterpret_cast<uint4*>(sA + off) = make_uint4(wh[0], wh[1], wh[2], wh[3]);
        *reinterpret_cast<uint4*>(sLo + off) = make_uint4(wl[0], wl[1], wl[2], wl[3]);
      }
    }
    fence_async_shared();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars.ds);
    if (ctl) {
      ok = wait(&bars.ds, i & 1);
      if (ok) {
        tc_fence_after();
        // dK from the hi half of dS alone (~1e-3 relative) when one launch holds every prototype;
        // over chunks of a larger set (dK sums more prototypes and grows with them) from both
        // halves. dQ, a sum over every token of every user, always takes both.
#pragma unroll
        for (int s = 0; s < KP / 16; ++s)
          umma_bf16(tb + CK, sw128_desc(smem_u32(sA) + (s / 4) * kBlk + (s % 4) * 32, 16, 1024),
                    sw128_desc(smem_u32(sQ) + s * 2048, QBLK, 1024), iV, s > 0);
        if constexpr (CHUNK) {
#pragma unroll
          for (int s = 0; s < KP / 16; ++s)
            umma_bf16(tb + CK, sw128_desc(smem_u32(sLo) + (s / 4) * kBlk + (s % 4) * 32, 16, 1024),
                      sw128_desc(smem_u32(sQ) + s * 2048, QBLK, 1024), iV, 1u);
        }
#pragma unroll
        for (int g = 0; g < QBLOCKS; ++g)
#pragma unroll
          for (int half = 0; half < 2; ++half)
#pragma unroll
            for (int s = 0; s < 8; ++s) {
              const uint32_t abase = smem_u32(half == 0 ? sA : sLo) + 2 * g * kBlk;
              umma_bf16(tb + CQ + g * D, sw128_desc(abase + s * 2048, kBlk, 1024),
                        sw128_desc(smem_u32(sK) + s * 2048, kBlk, 1024), iQ,
                        (fresh && half == 0 && s == 0) ? 0u : 1u);
            }
        umma_commit(&bars.m3);
      }
    }
    ok = __all_sync(0xffffffffu, wait(&bars.m3, i & 1));
    if (!ok) break;
    tc_fence_after();
    if (ctl && i + 1 < ntiles) {  // every MMA of this tile is complete: K, Q and dO are free
      if (tn.j == 0) load_qdo(tn);
      load_k(tn);
    }
    // dK (scaled) and dV rows: warpgroup wg holds channels [wg D/2, (wg+1) D/2) of token row r.
    // With 64 or more prototype columns per warpgroup the rows go out coalesced: each warp stages
    // its 32 rows x 32 channels (128 B a row) in the part of A hi / A lo that only it writes, and
    // reads them back so that one store covers four whole 128-byte rows.
    const int urows = (p.cu_seqlens[t.b + 1] - p.cu_seqlens[t.b]) - t.j * 128;  // this user's rows in the tile
    uint8_t* stk = sA + wg * (NCOL / 64) * kBlk + q4 * 32 * 128;   // this warp's staging (dK)
    uint8_t* stv = sLo + wg * (NCOL / 64) * kBlk + q4 * 32 * 128;  // (dV)
    auto stage_row = [&](uint8_t* st, const uint32_t* v, float mul) {  // lane's 32 floats -> row `lane`
#pragma unroll
      for (int ch = 0; ch < 8; ++ch)
        *reinterpret_cast<float4*>(st + lane * 128 + ((ch ^ (lane & 7)) << 4)) =
            make_float4(mul * __uint_as_float(v[4 * ch]), mul * __uint_as_float(v[4 * ch + 1]),
                        mul * __uint_as_float(v[4 * ch + 2]), mul * __uint_as_float(v[4 * ch + 3]));
    };
    auto staged = [&](const uint8_t* st, int u) -> float4 {  // row 4u + lane/8, chunk lane%8
      const int rho = 4 * u + (lane >> 3);
      return *reinterpret_cast<const float4*>(st + rho * 128 + (((lane & 7) ^ (rho & 7)) << 4));
    };
#pragma unroll
    for (int c = 0; c < D / 2; c += 32) {
      const int cc = wg * (D / 2) + c;
      uint32_t kr[32], vr[32];
      tmem_ld32(tb + loff + CK + cc, kr);
      tmem_ld32(tb + loff + CV + cc, vr);
      tmem_ld_wait();
      if constexpr (NCOL >= 64) {
        stage_row(stk, kr, p.scale);
        stage_row(stv, vr, 1.f);
        __syncwarp();
        if (accumulate) {
          // the previous chunks' values, all in flight together before any store (a load placed
          // after a store of the same arrays cannot be moved ahead of it)
          float4 pk[8], pv[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int row = q4 * 32 + 4 * u + (lane >> 3);
            const int64_t tk = static_cast<int64_t>(tok0) + row;
            const int64_t off = (tk * p.H + t.h) * D + cc + (lane & 7) * 4;
            const bool in = row < urows && tk < p.total_tokens;
            pk[u] = in ? *reinterpret_cast<const float4*>(p.dk + off) : make_float4(0.f, 0.f, 0.f, 0.f);
            pv[u] = in ? *reinterpret_cast<const float4*>(p.dv + off) : make_float4(0.f, 0.f, 0.f, 0.f);
          }
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int row = q4 * 32 + 4 * u + (lane >> 3);
            const int64_t tk = static_cast<int64_t>(tok0) + row;
            if (row < urows && tk < p.total_tokens) {
              const int64_t off = (tk * p.H + t.h) * D + cc + (lane & 7) * 4;
              float4 gk = staged(stk, u), gv = staged(stv, u);
              gk.x += pk[u].x; gk.y += pk[u].y; gk.z += pk[u].z; gk.w += pk[u].w;
              gv.x += pv[u].x; gv.y += pv[u].y; gv.z += pv[u].z; gv.w += pv[u].w;
              *reinterpret_cast<float4*>(p.dk + off) = gk;
              *reinterpret_cast<float4*>(p.dv + off) = gv;
            }
          }
        } else {
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int row = q4 * 32 + 4 * u + (lane >> 3);  // token row in the tile
            const int64_t tk = static_cast<int64_t>(tok0) + row;
            if (row < urows && tk < p.total_tokens) {
              const int64_t off = (tk * p.H + t.h) * D + cc + (lane & 7) * 4;
              *reinterpret_cast<float4*>(p.dk + off) = staged(stk, u);
              *reinterpret_cast<float4*>(p.dv + off) = staged(stv, u);
            }
          }
        }
        __syncwarp();
      } else {
        if (tok < p.total_tokens && (t.j * 128 + r) < (p.cu_seqlens[t.b + 1] - p.cu_seqlens[t.b])) {
          float* dk = p.dk + (static_cast<int64_t>(tok) * p.H + t.h) * D + cc;
          float* dv = p.dv + (static_cast<int64_t>(tok) * p.H + t.h) * D + cc;
#pragma unroll
          for (int u = 0; u < 32; u += 4) {
            float4 gk = make_float4(p.scale * __uint_as_float(kr[u]), p.scale * __uint_as_float(kr[u + 1]),
                                    p.scale * __uint_as_float(kr[u + 2]), p.scale * __uint_as_float(kr[u + 3]));
            float4 gv = make_float4(__uint_as_float(vr[u]), __uint_as_float(vr[u + 1]), __uint_as_float(vr[u + 2]),
                                    __uint_as_float(vr[u + 3]));
            if (accumulate) {
              const float4 pk = *reinterpret_cast<const float4*>(dk + u);
              const float4 pv = *reinterpret_cast<const float4*>(dv + u);
              gk.x += pk.x; gk.y += pk.y; gk.z += pk.z; gk.w += pk.w;
              gv.x += pv.x; gv.y += pv.y; gv.z += pv.z; gv.w += pv.w;
            }
            *reinterpret_cast<float4*>(dk + u) = gk;
            *reinterpret_cast<float4*>(dv + u) = gv;
          }
        }
      }
    }
    if (flush && wg < QBLOCKS) {
      // dQ block wg (prototypes 128 wg + r) of this segment, scaled, into its partial slot; only
      // this CTA writes the slot, and each element always by the same warp. Staged like dK.
      const int slot = (t.b * p.H + t.h) + static_cast<int>(blockIdx.x);
      const bool add = segt >= kDqFlush;
      float* qbase = p.dq_partial + (static_cast<int64_t>(slot) * p.k + wg * 128) * D;
#pragma unroll
      for (int c = 0; c < D; c += 32) {
        uint32_t qr[32];
        tmem_ld32(tb + loff + CQ + wg * D + c, qr);
        tmem_ld_wait();
        if constexpr (NCOL >= 64) {
          stage_row(stk, qr, p.scale);
          __syncwarp();
          float4 prev[8];  // all the slot's previous values in flight together
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int row = q4 * 32 + 4 * u + (lane >> 3);  // prototype within the block
            prev[u] = (add && wg * 128 + row < p.k)
                          ? *reinterpret_cast<const float4*>(qbase + static_cast<int64_t>(row) * D + c + (lane & 7) * 4)
                          : make_float4(0.f, 0.f, 0.f, 0.f);
          }
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int row = q4 * 32 + 4 * u + (lane >> 3);
            if (wg * 128 + row < p.k) {
              float4 o = staged(stk, u);
              o.x += prev[u].x;
              o.y += prev[u].y;
              o.z += prev[u].z;
              o.w += prev[u].w;
              *reinterpret_cast<float4*>(qbase + static_cast<int64_t>(row) * D + c + (lane & 7) * 4) = o;
            }
          }
          __syncwarp();
        } else {
          const int jrow = wg * 128 + r;
          if (jrow < p.k) {
            float* dst = qbase + static_cast<int64_t>(r) * D + c;
#pragma unroll
            for (int u = 0; u < 32; u += 4) {
              float4 o = make_float4(p.scale * __uint_as_float(qr[u]), p.scale * __uint_as_float(qr[u + 1]),
                                     p.scale * __uint_as_float(qr[u + 2]), p.scale * __uint_as_float(qr[u + 3]));
              if (add) {
                const float4 prev = *reinterpret_cast<const float4*>(dst + u);
                o.x += prev.x;
                o.y += prev.y;
                o.z += prev.z;
                o.w += prev.w;
              }
              *reinterpret_cast<float4*>(dst + u) = o;
            }
          }
        }
      }
    }
    tc_fence_before();
    __syncwarp();
    if (first) ++nseg;
    t = tn;
  }
  if (ctl) {
    umma_commit(&bars.drain);  // completes when every MMA issued above has
    wait(&bars.drain, 0, true);
    // on an early exit, loads issued for a tile that was not reached must land first
    if (nk_issued > nk_seen) wait(&bars.ldk, (nk_issued - 1) & 1, true);
    if (nv_issued > nv_seen) wait(&bars.ldv, (nv_issued - 1) & 1, true);
    if (nq_issued > nseg) wait(&bars.qd, (nq_issued - 1) & 1, true);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tb, 512);
  }
}

// dq[(b?) h] = sum over the segments it collects of their partial slots, fixed order.
__global__ void sa_bwd_dq_reduce(const SaBwdParams p, const SaBwdChunk ck, int D, float* __restrict__ dq) {
  const int64_t per = static_cast<int64_t>(p.k) * D;
  const int qsets = p.q_per_user ? p.B * p.H : p.H;
  const int64_t n = static_cast<int64_t>(qsets) * per;
  const int W = p.hdr->tiles_per_cluster;
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < n;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int qs = static_cast<int>(e / per);
    const int64_t within = e - static_cast<int64_t>(qs) * per;
    const int b0 = p.q_per_user ? qs / p.H : 0, b1 = p.q_per_user ? b0 + 1 : p.B;
    const int h = p.q_per_user ? qs % p.H : qs;
    float acc = 0.f;
    for (int b = b0; b < b1; ++b) {
      const int nb = p.tile_prefix[b + 1] - p.tile_prefix[b];
      if (nb == 0 || W == 0) continue;
      const int t0 = p.H * p.tile_prefix[b] + h * nb;
      const int s = b * p.H + h;
      for (int c = t0 / W; c <= (t0 + nb - 1) / W; ++c) acc += p.dq_partial[static_cast<int64_t>(s + c) * per + within];
    }
    dq[(static_cast<int64_t>(qs) * ck.kt + ck.j0) * D + within] = acc;
  }
}

// dK, dV rows of padding tokens (positions >= seqused inside a user) are zero.
__global__ void sa_bwd_zero_padding(const SaBwdParams p, int D) {
  const int b = blockIdx.x;
  const int64_t lo = p.cu_seqlens[b] + bwd_used(p, b);
  const int64_t hi = (static_cast<int64_t>(p.cu_seqlens[b + 1]) < p.total_tokens) ? p.cu_seqlens[b + 1] : p.total_tokens;
  // rows inside the last partial tile are written by the main kernel; zero from the next tile on
  const int64_t first_untouched = p.cu_seqlens[b] + ((bwd_used(p, b) + 127) / 128) * 128;
  const int64_t z0 = (lo > first_untouched) ? lo : first_untouched;
  for (int64_t i = z0 * p.H * D + threadIdx.x; i < hi * p.H * D; i += blockDim.x) {
    p.dk[i] = 0.f;
    p.dv[i] = 0.f;
  }
}

template <int D, int KP, bool CHUNK = false>
cudaError_t bwd_launch_t(int num_ctas, const CUtensorMap& mQ, const CUtensorMap& mDO, const CUtensorMap& mK,
                         const CUtensorMap& mV, const SaBwdParams& p, const SaBwdChunk& ck, cudaStream_t stream) {
  auto kern = sa_bwd_kernel<D, KP, CHUNK>;
  const size_t smem = bwd_layout(D, KP).total;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<num_ctas, kBwdThreads, smem, stream>>>(mQ, mDO, mK, mV, p, ck);
  return cudaGetLastError();
}

}  // namespace

namespace {
// One CTA holds all k prototypes of a tile (TMEM: S^T / dA^T, dV, dK and the dQ blocks).
bool bwd_one_launch(int D, int k) {
  if (D != 64 && D != 128) return false;
  if (!(k == 16 || k == 32 || k == 64 || k == 128 || k == 256)) return false;
  if (bwd_tmem_cols(D, k) + ((k + 31) / 32 * 32 - k) > 512) return false;
  return bwd_layout(D, k).total <= 227 * 1024;
}
}  // namespace

int sa_bwd_chunk(int D, int k) {
  if (bwd_one_launch(D, k)) return k;
  if (D != 64 && D != 128) return 0;
  const int c = (D == 128) ? 128 : 256;
  return (k > c && k % c == 0 && k <= kMaxChunkedProtos) ? c : 0;
}

bool sa_bwd_supported(int D, int k) { return sa_bwd_chunk(D, k) > 0; }

size_t sa_bwd_smem_bytes(int D, int k) { return bwd_layout(D, k).total; }

cudaError_t launch_sa_bwd(int D, int num_ctas, const CUtensorMap& mQ, const CUtensorMap& mDO,
                          const CUtensorMap& mK, const CUtensorMap& mV, const SaBwdParams& p,
                          const SaBwdChunk& ck, cudaStream_t stream) {
  const bool chunk = ck.kt != p.k;
  if (chunk && D == 64 && p.k == 256) return bwd_launch_t<64, 256, true>(num_ctas, mQ, mDO, mK, mV, p, ck, stream);
  if (chunk && D == 128 && p.k == 128) return bwd_launch_t<128, 128, true>(num_ctas, mQ, mDO, mK, mV, p, ck, stream);
  if (chunk) return cudaErrorInvalidValue;
#define SKA_BWD_CASE(DD, KK) \
  if (D == DD && p.k == KK) return bwd_launch_t<DD, KK>(num_ctas, mQ, mDO, mK, mV, p, ck, stream);
  SKA_BWD_CASE(64, 16)
  SKA_BWD_CASE(64, 32)
  SKA_BWD_CASE(64, 64)
  SKA_BWD_CASE(64, 128)
  SKA_BWD_CASE(64, 256)
  SKA_BWD_CASE(128, 16)
  SKA_BWD_CASE(128, 32)
  SKA_BWD_CASE(128, 64)
  SKA_BWD_CASE(128, 128)
#undef SKA_BWD_CASE
  return cudaErrorInvalidValue;
}

cudaError_t launch_sa_bwd_finish(const SaBwdParams& p, const SaBwdChunk& ck, int D, float* dq, cudaStream_t stream) {
  sa_bwd_dq_reduce<<<592, 256, 0, stream>>>(p, ck, D, dq);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (p.B > 0) sa_bwd_zero_padding<<<p.B, 256, 0, stream>>>(p, D);
  return cudaGetLastError();
}

}  // namespace ska
