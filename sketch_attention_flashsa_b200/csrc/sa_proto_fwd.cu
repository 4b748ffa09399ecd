// FlashSA forward with prototype-wise normalisation on sm_100a.
//
// SequenceO1 §3.1: S = scale Q K^T (Eq. (7)), A = softmax over the k prototypes for every
// history token (Eq. (8)), sketch = A V (Eq. (9)); §4.4 (FlashSA): one streaming pass over the
// history with block-wise affinities, softmax statistics and aggregation, never storing S.
//
// Layout of the computation (one cluster of CS CTAs works on one stream of 128-token tiles;
// CTA c of the cluster owns prototypes [c*KC, (c+1)*KC)):
//   MMA1  S^T[tok, j]  = K_tile[tok, :] . Q_c[j, :]^T     M=128 tokens, N=KC, K=D   (TMEM)
//   softmax threads own one token row each: max and sum over this CTA's KC prototypes, an
//         exchange of (max, sum) with the other CTAs of the cluster through distributed
//         shared memory, then P[tok, j] = exp(S - lse_tok) in bf16 to shared memory.
//   MMA2  O^T[dd, j]  += V_tile[tok, dd]^T . P[tok, j]    M=D, N=KC, K=128 tokens   (TMEM)
//         in fp16: P is rounded to fp16 (11 significant bits, eight times finer than bf16) and
//         the bf16 V tile is rewritten in place as fp16 (exact inside the fp16 range) by two
//         converter warps, so that the aggregation keeps ~5e-4 relative precision per weight.
// Tiles of all (user, head) segments are concatenated and split evenly over the persistent
// clusters; a cluster writes one fp32 partial sketch per segment it touches, and a second
// kernel sums the partials of each segment in a fixed order (a plain sum: each token's
// normalisation is complete inside the tile that holds it).
//
// Warp roles (384 threads): warp 0 = TMA producer, warp 1 = TMEM owner + MMA issuer,
// warps 2-3 = V converters, warps 4-11 = two softmax warpgroups (each owns half of the KC
// columns).
#include <cstdio>

#include "ska_internal.h"
#include "ska_proto_common.cuh"
#include "ska_ptx.cuh"

namespace ska {

namespace {

constexpr int kThreads = 384;
constexpr int kSoftmaxThreads = 256;
constexpr int kSoftmaxWarps = 8;
constexpr int kConvThreads = 64;
constexpr int kPrefetchTiles = 3;  // L2 prefetch distance of the producer, in tiles
constexpr int kSlotBytes = 16384;  // one [128 rows x 64 bf16] swizzled block
constexpr int kMaxRing = 8;

// Groups of four exponentials (out of every eight) computed on the FMA pipe by exp2_fma_pair
// instead of MUFU. At d = 128 the MUFU time of a tile equals its MMA time, but in this pipeline
// the softmax is bound by its dependency chain, not by MUFU throughput, and the longer unrolled
// loop costs instruction fetches: on the 8 x 100K x 8-head workload the fused kernel took
// 2.45 ms with no group on the FMA pipe, 2.65 ms with one and 2.77 ms with two, so it is off.
constexpr int kExpFmaGroups = 0;
__host__ __device__ constexpr bool exp_on_fma(int group4) { return (group4 & 7) < kExpFmaGroups; }

struct SmemLayout {
  uint32_t q_off, p_off, k_off, v_off, x_off, total;
};

__host__ __device__ inline SmemLayout smem_layout(int D, int KC, int CS, int nk, int nv) {
  SmemLayout L;
  uint32_t off = 0;
  L.q_off = off;
  off += KC * D * 2;  // Q_c, D/64 blocks of KC rows x 128 B
  off = (off + 1023) & ~1023u;
  L.p_off = off;
  off += ((KC + 63) / 64) * kSlotBytes;  // P, KC/64 blocks of 128 rows x 128 B
  L.k_off = off;
  off += nk * kSlotBytes;
  L.v_off = off;
  off += nv * (D / 64) * kSlotBytes;
  L.x_off = off;
  off += 2 * CS * 2 * 128 * 8;  // (max, sum) exchange: [parity][cta][wg][row]
  L.total = off;
  return L;
}

struct Bars {
  uint64_t kfull[kMaxRing], kempty[kMaxRing];
  uint64_t vfull[kMaxRing], vempty[kMaxRing], vconv[kMaxRing];
  uint64_t qfull, qfree, sfull, sfree, pfull, pfree, ofull, ofree, drain;
  uint64_t xbar[2];
  uint32_t tmem_base;
  int abort_flag;
};

// Segment epilogue (once per segment, kept out of line so that it does not crowd the softmax
// loop's instructions): this warp's rows of O^T, NCOL prototype columns of TMEM starting at tO,
// into the partial sketch dst[j * D + dd]. D = 128: lane row = channel; D = 64: lanes 0-15 of
// each quarter hold the channels (M = 64 accumulator layout).
template <int D, int NCOL>
__device__ __noinline__ void drain_o(uint32_t tO, float* dst, int q4, int lane) {
  tc_fence_after();
  const int dd = (D == 128) ? q4 * 32 + lane : ((lane < 16) ? q4 * 16 + lane : -1);
  for (int c = 0; c < NCOL; c += 8) {
    float ov[8];
    tmem_ld8(tO + c, reinterpret_cast<uint32_t*>(ov));
    tmem_ld_wait();
    if (dd >= 0) {
#pragma unroll
      for (int u = 0; u < 8; ++u) dst[(c + u) * D + dd] = ov[u];
    }
  }
  tc_fence_before();
  __syncwarp();
}

template <int D, int KC>
__global__ void __launch_bounds__(kThreads, 1)
    sa_proto_fwd_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapK,
                        const __grid_constant__ CUtensorMap mapV, const ProtoFwdParams p) {
  constexpr int KB = D / 64;        // 64-wide d blocks
  constexpr int NCOL = KC / 2;      // S columns per softmax thread
  constexpr int NALLOC = (2 * KC <= 32) ? 32 : (2 * KC <= 64) ? 64 : (2 * KC <= 128) ? 128 : (2 * KC <= 256) ? 256 : 512;
  static_assert(KC % 16 == 0 && KC <= 256, "KC");
  static_assert(NCOL % 8 == 0, "NCOL");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ Bars bars;

  const int CS = (int)cluster_nctarank();
  const int rank = (int)cluster_ctarank();
  const int cid = (int)cluster_id_x();
  const int ncl = (int)nclusters_x();
  const SmemLayout L = smem_layout(D, KC, CS, p.nk_slots, p.nv_entries);
  uint8_t* sQ = smem + L.q_off;
  uint8_t* sP = smem + L.p_off;
  uint8_t* sK = smem + L.k_off;
  uint8_t* sV = smem + L.v_off;
  float2* sX = reinterpret_cast<float2*>(smem + L.x_off);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < p.nk_slots; ++i) { mbar_init(&bars.kfull[i], 1); mbar_init(&bars.kempty[i], 1); }
    for (int i = 0; i < p.nv_entries; ++i) {
      mbar_init(&bars.vfull[i], 1);
      mbar_init(&bars.vempty[i], 1);
      mbar_init(&bars.vconv[i], kConvThreads);
    }
    mbar_init(&bars.qfull, 1);
    mbar_init(&bars.qfree, 1);
    mbar_init(&bars.sfull, 1);
    mbar_init(&bars.sfree, kSoftmaxWarps);
    mbar_init(&bars.pfull, kSoftmaxWarps);
    mbar_init(&bars.pfree, 1);
    mbar_init(&bars.ofull, 1);
    mbar_init(&bars.ofree, kSoftmaxWarps);
    mbar_init(&bars.drain, 1);
    mbar_init(&bars.xbar[0], 1);  // one arming arrival + CS * 256 * 8 transaction bytes
    mbar_init(&bars.xbar[1], 1);
    bars.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars.tmem_base, NALLOC);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  if (CS > 1) cluster_sync();
  tc_fence_after();
  const uint32_t tbase = bars.tmem_base;
  const uint32_t tS = tbase;        // S^T: 128 lanes x KC columns
  const uint32_t tO = tbase + KC;   // O^T: D rows x KC columns

  Waiter wait{&bars.abort_flag, &p.hdr->status, p.budget_ns};

  const int total = p.hdr->total_tiles;
  const int W = p.hdr->tiles_per_cluster;
  const int g0 = cid * W;
  const int g1 = min(total, g0 + W);
  const int ntiles = (W > 0 && g0 < total) ? (g1 - g0) : 0;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && ntiles > 0) {
      tma_prefetch_desc(&mapQ);
      tma_prefetch_desc(&mapK);
      tma_prefetch_desc(&mapV);
      TilePos tk, tv, tp;
      tile_seek(p, g0, tk);
      tv = tk;
      tp = tk;
      int ip = 0;  // next tile to prefetch into L2 (rank 0 of the cluster only)
      auto prefetch_to = [&](int upto) {
        while (ip < ntiles && ip < upto) {
          const int tok0 = p.cu_seqlens[tp.b] + tp.j * kTileTokens;
          for (int kb = 0; kb < KB; ++kb) {
            tma_prefetch_l2_2d(&mapK, tp.h * D + kb * 64, tok0);
            tma_prefetch_l2_2d(&mapV, tp.h * D + kb * 64, tok0);
          }
          ++ip;
          tile_next(p, tp);
        }
      };
      int kslot = 0, kuse = 0;  // K ring position, number of slot fills issued
      int vent = 0, vuse = 0;
      int nseg = 0;
      bool skip_first = (p.debug_flags & 1u) != 0;
      bool ok = true;
      for (int i = 0; i <= ntiles && ok; ++i) {
        if (rank == 0) prefetch_to(i + kPrefetchTiles);
        if (i < ntiles) {
          const bool first = (tk.j == 0) || (i == 0);
          if (first) {
            if (nseg > 0) ok = wait(&bars.qfree, (nseg - 1) & 1);
            if (!ok) break;
            const int row = (p.q_per_user ? tk.b * p.H * p.k : 0) + tk.h * p.k + rank * KC;
            mbar_expect_tx(&bars.qfull, KC * D * 2);
            for (int kb = 0; kb < KB; ++kb) tma_load_2d(sQ + kb * KC * 128, &mapQ, &bars.qfull, kb * 64, row);
            ++nseg;
          }
          const int tok0 = p.cu_seqlens[tk.b] + tk.j * kTileTokens;
          for (int kb = 0; kb < KB; ++kb) {
            const int slot = kslot;
            const int use = kuse / p.nk_slots;  // completed uses of this slot
            ok = wait(&bars.kempty[slot], (use & 1) ^ 1);
            if (!ok) break;
            if (skip_first) {
              skip_first = false;  // withhold this arrival: the MMA warp's wait must run out
            } else {
              mbar_expect_tx(&bars.kfull[slot], kSlotBytes);
              tma_load_2d(sK + slot * kSlotBytes, &mapK, &bars.kfull[slot], tk.h * D + kb * 64, tok0);
            }
            kslot = (kslot + 1 == p.nk_slots) ? 0 : kslot + 1;
            ++kuse;
          }
          if (!ok) break;
          tile_next(p, tk);
        }
        if (i >= 1) {
          const int use = vuse / p.nv_entries;
          ok = wait(&bars.vempty[vent], (use & 1) ^ 1);
          if (!ok) break;
          const int tok0 = p.cu_seqlens[tv.b] + tv.j * kTileTokens;
          mbar_expect_tx(&bars.vfull[vent], KB * kSlotBytes);
          for (int kb = 0; kb < KB; ++kb)
            tma_load_2d(sV + (vent * KB + kb) * kSlotBytes, &mapV, &bars.vfull[vent], tv.h * D + kb * 64, tok0);
          vent = (vent + 1 == p.nv_entries) ? 0 : vent + 1;
          ++vuse;
          tile_next(p, tv);
        }
      }
      // Drain: every load this thread issued must have landed before the CTA exits.
      for (int s = 0; s < p.nk_slots; ++s) {
        const int fills = (kuse > s) ? (kuse - s - 1) / p.nk_slots + 1 : 0;
        if (fills > 0) wait(&bars.kfull[s], (fills - 1) & 1, false, true);
      }
      for (int s = 0; s < p.nv_entries; ++s) {
        const int fills = (vuse > s) ? (vuse - s - 1) / p.nv_entries + 1 : 0;
        if (fills > 0) wait(&bars.vfull[s], (fills - 1) & 1, false, true);
      }
      if (nseg > 0) wait(&bars.qfull, (nseg - 1) & 1, false, true);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && ntiles > 0) {
      constexpr uint32_t idesc1 = idesc_bf16_f32(128, KC, false, false);
      constexpr uint32_t idesc2 = idesc_bf16_f32(D, KC, true, true, /*f16_inputs=*/true);
      TilePos t1, t2;
      tile_seek(p, g0, t1);
      t2 = t1;
      int kslot = 0, kuse = 0, vent = 0, vuse = 0;
      int nseg1 = 0, nseg2 = 0;
      bool ok = true;
      for (int i = 0; i <= ntiles && ok; ++i) {
        if (i < ntiles) {
          const bool first = (t1.j == 0) || (i == 0);
          const bool last = (t1.j == t1.nb - 1) || (i == ntiles - 1);
          if (first) {
            ok = wait(&bars.qfull, nseg1 & 1);
            if (!ok) break;
            ++nseg1;
          }
          if (i > 0) {
            ok = wait(&bars.sfree, (i - 1) & 1);
            if (!ok) break;
          }
          tc_fence_after();
          int slots[KB];
          for (int kb = 0; kb < KB; ++kb) {
            slots[kb] = kslot;
            ok = wait(&bars.kfull[kslot], (kuse / p.nk_slots) & 1);
            if (!ok) break;
            kslot = (kslot + 1 == p.nk_slots) ? 0 : kslot + 1;
            ++kuse;
          }
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int s = 0; s < D / 16; ++s) {
            const uint64_t ad = sw128_desc(smem_u32(sK + slots[s / 4] * kSlotBytes) + (s % 4) * 32, 16, 1024);
            const uint64_t bd = sw128_desc(smem_u32(sQ + (s / 4) * KC * 128) + (s % 4) * 32, 16, 1024);
            umma_bf16(tS, ad, bd, idesc1, s > 0 ? 1u : 0u);
          }
          for (int kb = 0; kb < KB; ++kb) umma_commit(&bars.kempty[slots[kb]]);
          umma_commit(&bars.sfull);
          if (last) umma_commit(&bars.qfree);
          tile_next(p, t1);
        }
        if (i >= 1) {
          const bool first = (t2.j == 0) || (i == 1);
          const bool last = (t2.j == t2.nb - 1) || (i == ntiles);
          ok = wait(&bars.pfull, (i - 1) & 1);
          if (!ok) break;
          ok = wait(&bars.vconv[vent], (vuse / p.nv_entries) & 1);
          if (!ok) break;
          if (first && nseg2 > 0) {
            ok = wait(&bars.ofree, (nseg2 - 1) & 1);
            if (!ok) break;
          }
          tc_fence_after();
          const uint32_t vbase = smem_u32(sV + vent * KB * kSlotBytes);
          const uint32_t pbase = smem_u32(sP);
#pragma unroll
          for (int s = 0; s < kTileTokens / 16; ++s) {
            const uint64_t ad = sw128_desc(vbase + s * 2048, kSlotBytes, 1024);
            const uint64_t bd = sw128_desc(pbase + s * 2048, kSlotBytes, 1024);
            umma_bf16(tO, ad, bd, idesc2, (first && s == 0) ? 0u : 1u);
          }
          umma_commit(&bars.vempty[vent]);
          umma_commit(&bars.pfree);
          if (last) {
            umma_commit(&bars.ofull);
            ++nseg2;
          }
          vent = (vent + 1 == p.nv_entries) ? 0 : vent + 1;
          ++vuse;
          tile_next(p, t2);
        }
      }
      // Drain every MMA this thread issued before TMEM is released.
      umma_commit(&bars.drain);
      wait(&bars.drain, 0, false, true);
    }
  } else if (warp == 2 || warp == 3) {
    // ------------------------------------------------------------ V converters: bf16 -> fp16
    const int ct = threadIdx.x - 64;
    int vent = 0, vuse = 0;
    bool ok = true;
    for (int i = 0; i < ntiles && ok; ++i) {
      ok = __all_sync(0xffffffffu, wait(&bars.vfull[vent], (vuse / p.nv_entries) & 1));
      if (!ok) break;
      uint4* base = reinterpret_cast<uint4*>(sV + vent * KB * kSlotBytes);
      constexpr int kChunks = KB * kSlotBytes / 16;
#pragma unroll 8
      for (int c = ct; c < kChunks; c += kConvThreads) {
        uint4 w = base[c];
        w.x = bf16x2_to_f16x2(w.x);
        w.y = bf16x2_to_f16x2(w.y);
        w.z = bf16x2_to_f16x2(w.z);
        w.w = bf16x2_to_f16x2(w.w);
        base[c] = w;
      }
      fence_async_shared();
      mbar_arrive(&bars.vconv[vent]);
      vent = (vent + 1 == p.nv_entries) ? 0 : vent + 1;
      ++vuse;
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax warpgroups
    const int g = (warp - 4) >> 2;          // warpgroup: columns [g*NCOL, (g+1)*NCOL)
    const int q4 = warp & 3;                // TMEM lane quarter
    const int r = q4 * 32 + lane;           // token row of this thread
    const int col0 = g * NCOL;
    const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
    const float c2 = p.scale_log2;
    const uint64_t c2x2 = f2_pack(c2, c2);
    TilePos t;
    if (ntiles > 0) tile_seek(p, g0, t);
    int nseg = 0;
    bool ok = true;
    const uint32_t xbase = smem_u32(sX);
    const uint32_t xbar_local[2] = {smem_u32(&bars.xbar[0]), smem_u32(&bars.xbar[1])};
    const bool x_owner = (threadIdx.x == 128);  // arms the exchange barrier's byte count
    constexpr uint32_t kXBytesPerCta = kSoftmaxThreads * 8;
    int cur_b = -1, used = 0, tok_base = 0;
    for (int i = 0; i < ntiles && ok; ++i) {
      if (t.b != cur_b) {
        cur_b = t.b;
        used = user_used(p, t.b);
        tok_base = p.cu_seqlens[t.b];
      }
      const int nvalid = min(kTileTokens, used - t.j * kTileTokens);
      const bool valid = r < nvalid;
      const int tok = tok_base + t.j * kTileTokens + r;
      const bool last = (t.j == t.nb - 1) || (i == ntiles - 1);
      const int par = i & 1;
      if (x_owner) mbar_expect_tx(&bars.xbar[par], kXBytesPerCta * CS);

      ok = __all_sync(0xffffffffu, wait(&bars.sfull, i & 1));
      if (!ok) break;
      tc_fence_after();
      uint32_t sv[NCOL];
      constexpr int R32 = (NCOL / 32) * 32;
      constexpr int R16 = R32 + ((NCOL - R32) >= 16 ? 16 : 0);
#pragma unroll
      for (int c = 0; c < R32; c += 32) tmem_ld32(tS + lane_off + col0 + c, sv + c);
      if constexpr (R16 > R32) tmem_ld16(tS + lane_off + col0 + R32, sv + R32);
      if constexpr (NCOL > R16) tmem_ld8(tS + lane_off + col0 + R16, sv + R16);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.sfree);

      // Local statistics in the log2 domain: m2 = max_j s_j * c2, l = sum_j 2^(s_j c2 - m2).
      // Four independent max chains and two packed-pair sum chains keep latency off the path.
      float m2 = -INFINITY, lsum = 0.f;
      if (valid) {
        float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
#pragma unroll
        for (int c = 0; c < NCOL; c += 8) {
          mx0 = max3f(mx0, __uint_as_float(sv[c + 0]), __uint_as_float(sv[c + 1]));
          mx1 = max3f(mx1, __uint_as_float(sv[c + 2]), __uint_as_float(sv[c + 3]));
          mx2 = max3f(mx2, __uint_as_float(sv[c + 4]), __uint_as_float(sv[c + 5]));
          mx3 = max3f(mx3, __uint_as_float(sv[c + 6]), __uint_as_float(sv[c + 7]));
        }
        m2 = fmaxf(max3f(mx0, mx1, mx2), mx3) * c2;
        const uint64_t negm = f2_pack(-m2, -m2);
        uint64_t acc0 = f2_pack(0.f, 0.f), acc1 = acc0;
#pragma unroll
        for (int c = 0; c < NCOL; c += 4) {
          float x0, x1, x2, x3;
          f2_unpack(f2_fma(f2_pack(__uint_as_float(sv[c]), __uint_as_float(sv[c + 1])), c2x2, negm), x0, x1);
          f2_unpack(f2_fma(f2_pack(__uint_as_float(sv[c + 2]), __uint_as_float(sv[c + 3])), c2x2, negm), x2, x3);
          float e0, e1, e2, e3;
          if (exp_on_fma(c / 4)) {
            exp2_fma_pair(x0, x1, e0, e1);
            exp2_fma_pair(x2, x3, e2, e3);
          } else {
            e0 = ex2_approx(x0);
            e1 = ex2_approx(x1);
            e2 = ex2_approx(x2);
            e3 = ex2_approx(x3);
          }
          sv[c] = __float_as_uint(e0);
          sv[c + 1] = __float_as_uint(e1);
          sv[c + 2] = __float_as_uint(e2);
          sv[c + 3] = __float_as_uint(e3);
          acc0 = f2_add(acc0, f2_pack(e0, e1));
          acc1 = f2_add(acc1, f2_pack(e2, e3));
        }
        float a0, a1, b0, b1;
        f2_unpack(acc0, a0, a1);
        f2_unpack(acc1, b0, b1);
        lsum = (a0 + a1) + (b0 + b1);
      }
      // Exchange (m2, l) with every warpgroup of every CTA of the cluster: asynchronous
      // stores that count as transaction bytes on the destination CTA's exchange barrier.
      const uint32_t xoff = static_cast<uint32_t>((((par * CS + rank) * 2 + g) * 128 + r) * 8);
      for (int c = 0; c < CS; ++c)
        st_async_f32x2(mapa_shared(xbase + xoff, c), m2, lsum, mapa_shared(xbar_local[par], c));
      ok = __all_sync(0xffffffffu, wait(&bars.xbar[par], (i >> 1) & 1, true));
      if (!ok) break;
      // (unrolled so that the loads of a row's entries are in flight together)
      float M = -INFINITY;
#pragma unroll 4
      for (int c = 0; c < CS * 2; ++c) M = fmaxf(M, sX[(par * CS * 2 + c) * 128 + r].x);
      float Lsum = 0.f;
#pragma unroll 4
      for (int c = 0; c < CS * 2; ++c) {
        const float2 e = sX[(par * CS * 2 + c) * 128 + r];
        Lsum = fmaf(e.y, ex2_approx(e.x - M), Lsum);
      }
      const float f = valid ? __fdividef(ex2_approx(m2 - M), Lsum) : 0.f;
      const uint64_t f2 = f2_pack(f, f);

      // P[tok, j] = A_{j,tok} as fp16 into the swizzled MN-major operand of MMA2.
      if (i > 0) {
        ok = __all_sync(0xffffffffu, wait(&bars.pfree, (i - 1) & 1));
        if (!ok) break;
      }
#pragma unroll
      for (int c = 0; c < NCOL; c += 8) {
        const int jj = col0 + c;
        uint4 w;
        float a0, a1;
        f2_unpack(f2_mul(f2_pack(__uint_as_float(sv[c + 0]), __uint_as_float(sv[c + 1])), f2), a0, a1);
        w.x = pack_f16x2(a0, a1);
        f2_unpack(f2_mul(f2_pack(__uint_as_float(sv[c + 2]), __uint_as_float(sv[c + 3])), f2), a0, a1);
        w.y = pack_f16x2(a0, a1);
        f2_unpack(f2_mul(f2_pack(__uint_as_float(sv[c + 4]), __uint_as_float(sv[c + 5])), f2), a0, a1);
        w.z = pack_f16x2(a0, a1);
        f2_unpack(f2_mul(f2_pack(__uint_as_float(sv[c + 6]), __uint_as_float(sv[c + 7])), f2), a0, a1);
        w.w = pack_f16x2(a0, a1);
        if (!valid) w = make_uint4(0, 0, 0, 0);
        uint8_t* dst = sP + (jj >> 6) * kSlotBytes + sw128_offset(r, (jj & 63) * 2);
        *reinterpret_cast<uint4*>(dst) = w;
      }
      fence_async_shared();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.pfull);

      if (p.lse && valid && g == 0 && rank == 0 && tok < p.total_tokens)
        p.lse[static_cast<int64_t>(tok) * p.H + t.h] = (M + __log2f(Lsum)) * 0.69314718055994531f;

      if (last) {
        // Segment epilogue: O^T (this CTA's KC prototypes) -> partial sketch slot.
        ok = __all_sync(0xffffffffu, wait(&bars.ofull, nseg & 1));
        if (!ok) break;
        const int slot = (t.b * p.H + t.h) + cid;
        drain_o<D, NCOL>(tO + lane_off + col0, p.partial + (static_cast<int64_t>(slot) * p.k + rank * KC + col0) * D,
                         q4, lane);
        if (lane == 0) mbar_arrive(&bars.ofree);
        ++nseg;
      }
      tile_next(p, t);
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (CS > 1) cluster_sync();  // no CTA leaves while a peer may still write into it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, NALLOC);
  }
}

template <int D, int KC>
cudaError_t launch_t(const ProtoFwdLaunch& L, const CUtensorMap& mQ, const CUtensorMap& mK,
                     const CUtensorMap& mV, const ProtoFwdParams& p, cudaStream_t stream) {
  auto kern = sa_proto_fwd_kernel<D, KC>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.smem_bytes);
  if (e != cudaSuccess) return e;
  if (L.cluster > 1) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(L.num_clusters * L.cluster, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = L.smem_bytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = L.cluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, mQ, mK, mV, p);
}

}  // namespace

bool proto_fwd_plan(int D, int k, int num_sms, ProtoFwdLaunch* out, int* nk_slots, int* nv_entries) {
  if (D != 64 && D != 128) return false;
  if (k < 16 || k % 16 != 0) return false;
  const int cs = (k + kMaxProtosPerCta - 1) / kMaxProtosPerCta;
  if (cs > 8 || k % cs != 0) return false;
  const int kc = k / cs;
  if (kc % 16 != 0) return false;
  if (!(kc == 16 || kc == 32 || kc == 64 || kc == 128 || kc == 192 || kc == 256)) return false;
  // Fill shared memory: prefer deep rings for K (16 KB slots) and V (tile entries).
  const size_t budget = 227 * 1024 - 1024 /* alignment slack */ - 512 /* static */;
  const int kb = D / 64;
  int best_nk = 0, best_nv = 0;
  for (int nv = 1; nv <= kMaxRing; ++nv) {
    for (int nk = kb; nk <= kMaxRing; ++nk) {
      SmemLayout L = smem_layout(D, kc, cs, nk, nv);
      if (L.total > budget) continue;
      // score: balanced depth first (tiles of K and of V), then bytes, K before V
      const int score = min(nk / kb, nv) * 10000 + (nk + nv * kb) * 10 + (nk / kb >= nv ? 1 : 0);
      const int best = min(best_nk / kb, best_nv) * 10000 + (best_nk + best_nv * kb) * 10 +
                       (best_nk / kb >= best_nv ? 1 : 0);
      if (best_nk == 0 || score > best) { best_nk = nk; best_nv = nv; }
    }
  }
  if (best_nk == 0) return false;
  out->cluster = cs;
  out->kc = kc;
  out->num_clusters = num_sms / cs;
  out->smem_bytes = smem_layout(D, kc, cs, best_nk, best_nv).total + 1024;
  *nk_slots = best_nk;
  *nv_entries = best_nv;
  return true;
}

cudaError_t launch_proto_fwd(int D, const ProtoFwdLaunch& L, const CUtensorMap& mQ, const CUtensorMap& mK,
                             const CUtensorMap& mV, const ProtoFwdParams& p, cudaStream_t stream) {
#define SKA_PROTO_CASE(DD, KK) \
  if (D == DD && L.kc == KK) return launch_t<DD, KK>(L, mQ, mK, mV, p, stream);
  SKA_PROTO_CASE(64, 16)
  SKA_PROTO_CASE(64, 32)
  SKA_PROTO_CASE(64, 64)
  SKA_PROTO_CASE(64, 128)
  SKA_PROTO_CASE(64, 192)
  SKA_PROTO_CASE(64, 256)
  SKA_PROTO_CASE(128, 16)
  SKA_PROTO_CASE(128, 32)
  SKA_PROTO_CASE(128, 64)
  SKA_PROTO_CASE(128, 128)
  SKA_PROTO_CASE(128, 192)
  SKA_PROTO_CASE(128, 256)
#undef SKA_PROTO_CASE
  return cudaErrorInvalidValue;
}

}  // namespace ska
