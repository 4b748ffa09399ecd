// FlashSA forward with prototype-wise normalisation on sm_100a.
//
// SequenceO1 §3.1: S = scale Q K^T (Eq. (7)), A = softmax over the k prototypes for every
// history token (Eq. (8)), sketch = A V (Eq. (9)); §4.4 (FlashSA): one streaming pass over the
// history with block-wise affinities, softmax statistics and aggregation, never storing S.
//
// One cluster of CS CTAs works on one stream of 128-token tiles; CTA c owns the KC = k / CS
// prototypes [c KC, (c + 1) KC). The normalisation of a token is split into a part that is
// local to a CTA and a per-token factor folded into the values:
//   A[j, i] = E_c[i, j] * f_c[i],   E_c[i, j] = 2^(s_ij - m_c,i),   f_c[i] = 2^(m_c,i - M_i) / L_i
// with m_c,i the max of token i's scores (log2 units) over CTA c's prototypes, M_i the max over
// all k and L_i = sum_c 2^(m_c,i - M_i) sum_{j in c} E_c[i, j]. Hence
//   sketch_c = A_c V = E_c^T (f_c V):
// the softmax threads never wait for the other CTAs, and the cluster exchange of (m, l) feeds
// the warps that scale the value rows.
//   MMA1  S^T[tok, j] = K_tile[tok, :] . Q_c[j, :]^T      M=128 tokens, N=KC, K=D   (TMEM)
//   softmax warps (thread = token row, warpgroup = half of the KC columns): the row max over
//         the CTA's columns (the two warpgroups agree on it through shared memory), E in fp16
//         into shared memory (the MN-major B operand of MMA2), the row sums l; (m, l) go to
//         every CTA of the cluster as asynchronous stores counted on its exchange barrier.
//   converter warps (thread = token row): M, L and f_c of the row from the exchange, the lse,
//         and the bf16 V row rewritten in place as fp16 f_c * v (11 significant bits).
//   MMA2  O^T[dd, j] += V'[tok, dd]^T . E[tok, j]         M=D, N=KC, K=128 tokens   (TMEM, fp16)
//   mass  (optional) mass[j] += sum_tok f_c[tok] E[tok, j] as a fourth MMA with M=64 whose A
//         operand is a block holding f_c in its first row.
// Tiles of all (user, head) segments are concatenated and split evenly over the persistent
// clusters; a cluster writes one fp32 partial sketch per segment it touches, and a second
// kernel sums the partials of each segment in a fixed order (a plain sum: each token's
// normalisation is complete inside the tile that holds it).
//
// Warp roles (512 threads): warp 0 = TMA producer of Q and K, warp 1 = TMEM owner + MMA issuer,
// warp 2 = TMA producer of V, warps 4-7 = converters, warps 8-15 = two softmax warpgroups.
// Warpgroup 0 runs with 64 registers a thread, the converters with 48, the softmax warpgroups
// with 200.
#include <cstdio>
#include <mutex>

#include <cuda_fp16.h>

#include "ska_internal.h"
#include "ska_proto_common.cuh"
#include "ska_ptx.cuh"

namespace ska {

namespace {

constexpr int kThreads = 512;
constexpr int kSoftmaxWarps = 8;
constexpr int kConvWarps = 4;
constexpr int kSlotBytes = 16384;  // one [128 rows x 64 16-bit] swizzled block
constexpr int kMaxRing = 8;
// Exchange slots: tile i uses slot i mod 4. A CTA posts tile t only after its own converters
// finished tile t - 2, which needed every peer's post of tile t - 2, which each peer made only
// after its converters finished tile t - 4; so slot t mod 4 of every peer is free again.
constexpr int kXSlots = 4;
// The mass accumulator restarts every kMassChain tiles and its chains are summed in fp32 in shared
// memory: the tensor core's fp32 accumulation does not round to nearest, and positive terms summed
// in one chain drift low. Measured on 2 x 100K tokens, k = 512: chains of 16 tiles gave a sum over
// the prototypes 1.2e-5 (relative) below the token count; the bias scales with the chain length.
constexpr int kMassChain = 8;
// Registers per thread after the split (the launch gives 128 to each of the 512 threads): the
// producer / MMA warpgroup 64, the converters 48, the two softmax warpgroups 200 (the only
// split found without spills in any instantiation).
constexpr uint32_t kRoleRegs = 64;
constexpr uint32_t kConvRegs = 48;
constexpr uint32_t kSoftmaxRegs = 200;
static_assert(128 * kRoleRegs + 128 * kConvRegs + 256 * kSoftmaxRegs <= 65536, "register split");

struct Bars {
  uint64_t kfull[kMaxRing], kempty[kMaxRing];
  uint64_t vfull[kMaxRing], vempty[kMaxRing], vconv[kMaxRing];
  uint64_t qfull, qfree, sfull, sfree, pfull, pfree, ofull, ofree, drain;
  uint64_t xbar[kXSlots], mxbar[2], mfull, mfree;
  uint32_t tmem_base;
  int abort_flag;
};

struct SmemLayout {
  uint32_t q_off, p_off, k_off, v_off, x_off, m_off, ms_off, bar_off, total;
};

// Everything lives in the dynamic region, whose base is 1024-byte aligned when the kernel has no
// static shared memory.
__host__ __device__ inline SmemLayout smem_layout(int D, int KC, int CS, int nk, int nv, bool mass) {
  SmemLayout L;
  uint32_t off = 0;
  L.q_off = off;
  off += KC * D * 2;  // Q_c: D/64 blocks of KC rows x 128 B
  off = (off + 1023) & ~1023u;
  L.p_off = off;
  off += ((KC + 63) / 64) * kSlotBytes;  // E: KC/64 blocks of 128 token rows x 128 B
  L.k_off = off;
  off += nk * kSlotBytes;  // K ring: 64-channel blocks of a tile
  L.v_off = off;
  off += nv * (D / 64 + (mass ? 1 : 0)) * kSlotBytes;  // V entries (+ the factor block)
  L.x_off = off;
  off += kXSlots * CS * 2 * 128 * 8;  // (m, l) exchange: [slot][cta][warpgroup][row]
  L.m_off = off;
  off += 2 * 2 * 128 * 4;  // row max of each warpgroup: [parity][warpgroup][row]
  L.ms_off = off;
  off += mass ? KC * 4 : 0;  // fp32 sum of the mass chains of the current segment
  L.bar_off = off;
  off += (sizeof(Bars) + 15) & ~15u;
  L.total = off;
  return L;
}

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

template <int D, int KC, bool MASS>
__global__ void __launch_bounds__(kThreads, 1)
    sa_proto_fwd_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapK,
                        const __grid_constant__ CUtensorMap mapV, const ProtoFwdParams p) {
  constexpr int KB = D / 64;            // 64-channel blocks of a K or V tile
  constexpr int VB = KB + (MASS ? 1 : 0);  // blocks of a V entry
  constexpr int NCOL = KC / 2;          // S columns per softmax thread
  constexpr int NUSE = (MASS ? 3 : 2) * KC;
  constexpr int NALLOC = (NUSE <= 32) ? 32 : (NUSE <= 64) ? 64 : (NUSE <= 128) ? 128 : (NUSE <= 256) ? 256 : 512;
  static_assert(KC % 16 == 0 && KC <= 256, "KC");
  static_assert(NCOL % 8 == 0, "NCOL");
  static_assert(NUSE <= 512, "TMEM");

  extern __shared__ __align__(1024) uint8_t smem[];
  const int CS = (int)cluster_nctarank();
  const int rank = (int)cluster_ctarank();
  const int cid = (int)cluster_id_x();
  const SmemLayout L = smem_layout(D, KC, CS, p.nk_slots, p.nv_entries, MASS);
  Bars& bars = *reinterpret_cast<Bars*>(smem + L.bar_off);
  if ((smem_u32(smem) & 1023u) != 0) {  // the swizzled operands need a 1024-byte aligned base
    if (threadIdx.x == 0) atomicCAS(&p.hdr->status, 0, (int)SKA_ERR_UNSUPPORTED);
    return;  // uniform over the cluster: every CTA sees the same base
  }
  uint8_t* sQ = smem + L.q_off;
  uint8_t* sP = smem + L.p_off;
  uint8_t* sK = smem + L.k_off;
  uint8_t* sV = smem + L.v_off;
  float2* sX = reinterpret_cast<float2*>(smem + L.x_off);
  float* sM = reinterpret_cast<float*>(smem + L.m_off);
  float* sMass = reinterpret_cast<float*>(smem + L.ms_off);
  constexpr uint32_t kXBytesPerTile = 2 * 128 * 8;  // posted by one CTA into every CTA

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < p.nk_slots; ++i) { mbar_init(&bars.kfull[i], 1); mbar_init(&bars.kempty[i], 1); }
    for (int i = 0; i < p.nv_entries; ++i) {
      mbar_init(&bars.vfull[i], 1);
      mbar_init(&bars.vempty[i], 1);
      mbar_init(&bars.vconv[i], kConvWarps);
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
    mbar_init(&bars.mxbar[0], kSoftmaxWarps);
    mbar_init(&bars.mxbar[1], kSoftmaxWarps);
    mbar_init(&bars.mfull, 1);
    mbar_init(&bars.mfree, 2);  // the lane-quarter-0 warp of each softmax warpgroup
    // Exchange barriers: one arming arrival (with the expected bytes of all CS CTAs) per phase.
    // The first phase of every slot is armed here; a converter re-arms a slot as it consumes it.
    for (int s = 0; s < kXSlots; ++s) {
      mbar_init(&bars.xbar[s], 1);
      mbar_expect_tx(&bars.xbar[s], kXBytesPerTile * CS);
    }
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
  const uint32_t tS = tbase;           // S^T: 128 lanes x KC columns
  const uint32_t tO = tbase + KC;      // O^T: D rows x KC columns
  const uint32_t tMs = tbase + 2 * KC; // mass: M = 64 accumulator, row 0 used

  Waiter wait{&bars.abort_flag, &p.hdr->status, p.budget_ns};

  const int total = p.hdr->total_tiles;
  const int W = p.hdr->tiles_per_cluster;
  const int g0 = cid * W;
  const int g1 = min(total, g0 + W);
  const int ntiles = (W > 0 && g0 < total) ? (g1 - g0) : 0;

  // Each role's register budget is set inside its own branch, so that the compiler allocates the
  // code of that branch against it.
  if (warp < 4) {
   setmaxnreg_dec<kRoleRegs>();
   if (warp == 0) {
    // ------------------------------------------------------------ TMA producer: Q and K
    if (lane == 0 && ntiles > 0) {
      // No prefetch of later tiles into L2: on 8 x 100K x 8 heads, TMA prefetches of K and V three
      // or eight tiles ahead (2.03-2.05 ms) and prefetch instructions two to six tiles ahead
      // (2.09-2.10 ms) were both slower than none (1.98-1.99 ms).
      tma_prefetch_desc(&mapQ);
      tma_prefetch_desc(&mapK);
      tma_prefetch_desc(&mapV);
      TilePos tk;
      tile_seek(p, g0, tk);
      int kslot = 0, kuse = 0, nseg = 0;
      bool skip_first = (p.debug_flags & 1u) != 0;
      bool ok = true;
      for (int i = 0; i < ntiles && ok; ++i) {
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
          const int use = kuse / p.nk_slots;  // completed uses of this slot
          ok = wait(&bars.kempty[kslot], (use & 1) ^ 1);
          if (!ok) break;
          if (skip_first) {
            skip_first = false;  // withhold this arrival: the MMA warp's wait must run out
          } else {
            mbar_expect_tx(&bars.kfull[kslot], kSlotBytes);
            tma_load_2d(sK + kslot * kSlotBytes, &mapK, &bars.kfull[kslot], tk.h * D + kb * 64, tok0);
          }
          kslot = (kslot + 1 == p.nk_slots) ? 0 : kslot + 1;
          ++kuse;
        }
        tile_next(p, tk);
      }
      // Drain: every load this thread issued must have landed before the CTA exits.
      for (int s = 0; s < p.nk_slots; ++s) {
        const int fills = (kuse > s) ? (kuse - s - 1) / p.nk_slots + 1 : 0;
        if (fills > 0) wait(&bars.kfull[s], (fills - 1) & 1, false, true);
      }
      if (nseg > 0) wait(&bars.qfull, (nseg - 1) & 1, false, true);
    }
   } else if (warp == 2) {
    // ------------------------------------------------------------ TMA producer: V
    if (lane == 0 && ntiles > 0) {
      TilePos tv;
      tile_seek(p, g0, tv);
      int vent = 0, vuse = 0;
      bool ok = true;
      for (int i = 0; i < ntiles && ok; ++i) {
        ok = wait(&bars.vempty[vent], ((vuse / p.nv_entries) & 1) ^ 1);
        if (!ok) break;
        const int tok0 = p.cu_seqlens[tv.b] + tv.j * kTileTokens;
        mbar_expect_tx(&bars.vfull[vent], KB * kSlotBytes);
        for (int kb = 0; kb < KB; ++kb)
          tma_load_2d(sV + (vent * VB + kb) * kSlotBytes, &mapV, &bars.vfull[vent], tv.h * D + kb * 64, tok0);
        vent = (vent + 1 == p.nv_entries) ? 0 : vent + 1;
        ++vuse;
        tile_next(p, tv);
      }
      for (int s = 0; s < p.nv_entries; ++s) {
        const int fills = (vuse > s) ? (vuse - s - 1) / p.nv_entries + 1 : 0;
        if (fills > 0) wait(&bars.vfull[s], (fills - 1) & 1, false, true);
      }
    }
   } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && ntiles > 0) {
      constexpr uint32_t idesc1 = idesc_bf16_f32(128, KC, false, false);
      constexpr uint32_t idesc2 = idesc_bf16_f32(D, KC, true, true, /*f16_inputs=*/true);
      constexpr uint32_t idescm = idesc_bf16_f32(64, KC, true, true, /*f16_inputs=*/true);
      TilePos t1, t2;
      tile_seek(p, g0, t1);
      t2 = t1;
      int kslot = 0, kuse = 0, vent = 0, vuse = 0;
      int nseg1 = 0, nseg2 = 0;
      int sl2 = 0, nmc = 0;  // tile index inside the segment's part, mass chains completed
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
          const uint32_t vbase = smem_u32(sV + vent * VB * kSlotBytes);
          const uint32_t pbase = smem_u32(sP);
#pragma unroll
          for (int s = 0; s < kTileTokens / 16; ++s) {
            const uint64_t ad = sw128_desc(vbase + s * 2048, kSlotBytes, 1024);
            const uint64_t bd = sw128_desc(pbase + s * 2048, kSlotBytes, 1024);
            umma_bf16(tO, ad, bd, idesc2, (first && s == 0) ? 0u : 1u);
          }
          bool mend = false;
          if constexpr (MASS) {
            sl2 = first ? 0 : sl2 + 1;
            const bool mstart = (sl2 % kMassChain) == 0;
            mend = last || (sl2 % kMassChain) == kMassChain - 1;
            if (mstart && nmc > 0) {  // the previous chain has been read out of TMEM
              ok = wait(&bars.mfree, (nmc - 1) & 1);
              if (!ok) break;
              tc_fence_after();
            }
            const uint32_t fbase = vbase + KB * kSlotBytes;
#pragma unroll
            for (int s = 0; s < kTileTokens / 16; ++s) {
              const uint64_t ad = sw128_desc(fbase + s * 2048, kSlotBytes, 1024);
              const uint64_t bd = sw128_desc(pbase + s * 2048, kSlotBytes, 1024);
              umma_bf16(tMs, ad, bd, idescm, (mstart && s == 0) ? 0u : 1u);
            }
          }
          umma_commit(&bars.vempty[vent]);
          umma_commit(&bars.pfree);
          if (last) {
            umma_commit(&bars.ofull);
            ++nseg2;
          }
          if (mend) {
            umma_commit(&bars.mfull);
            ++nmc;
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
   }
  } else if (warp < 8) {
    setmaxnreg_dec<kConvRegs>();
    // ------------------------------------------------------------ converters: f * v -> fp16
    const int r = threadIdx.x - 128;  // token row of this thread
    const int sw = r & 7;             // 128-byte swizzle of the row: chunk c sits at c ^ sw
    if constexpr (MASS) {
      // The factor blocks hold f in element 0 of every row and zeros elsewhere (set once).
      for (int e = 0; e < p.nv_entries; ++e) {
        uint8_t* row = sV + (e * VB + KB) * kSlotBytes + r * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4*>(row + ((c ^ sw) << 4)) = make_uint4(0, 0, 0, 0);
      }
    }
    TilePos t;
    if (ntiles > 0) tile_seek(p, g0, t);
    int vent = 0, vuse = 0;
    int cur_b = -1, used = 0, tok_base = 0;
    bool ok = true;
    for (int i = 0; i < ntiles && ok; ++i) {
      if (t.b != cur_b) {
        cur_b = t.b;
        used = user_used(p, t.b);
        tok_base = p.cu_seqlens[t.b];
      }
      const bool valid = r < used - t.j * kTileTokens;
      const int tok = tok_base + t.j * kTileTokens + r;
      const int xs = i & (kXSlots - 1);
      ok = __all_sync(0xffffffffu, wait(&bars.xbar[xs], (i / kXSlots) & 1, true));
      if (!ok) break;
      // The row's global max M, total L and this CTA's factor f. Entry ((xs, c, g), r) holds the
      // (m, l) that warpgroup g of CTA c posted; both warpgroups of a CTA post the same m.
      const float2* xe = sX + static_cast<size_t>(xs) * CS * 2 * 128 + r;
      float M = -INFINITY;
#pragma unroll
      for (int c = 0; c < 8; ++c)
        if (c < CS) M = fmaxf(M, xe[(c * 2) * 128].x);
      float Lsum = 0.f, mown = 0.f;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        if (c < CS) {
          const float2 a = xe[(c * 2) * 128], b = xe[(c * 2 + 1) * 128];
          Lsum = fmaf(a.y + b.y, ex2_approx(a.x - M), Lsum);
          if (c == rank) mown = a.x;
        }
      }
      const float f = valid ? __fdividef(ex2_approx(mown - M), Lsum) : 0.f;
      if (threadIdx.x == 128) mbar_expect_tx(&bars.xbar[xs], kXBytesPerTile * CS);  // arms tile i + 4
      if (p.lse && valid && rank == 0 && tok < p.total_tokens)
        p.lse[static_cast<int64_t>(tok) * p.H + t.h] = (M + __log2f(Lsum)) * 0.69314718055994531f;
      // the token's largest weight over all k prototypes is 2^(M - M) / L
      if (p.maxw && valid && rank == 0 && tok < p.total_tokens)
        p.maxw[static_cast<int64_t>(tok) * p.H + t.h] = 1.f / Lsum;

      ok = __all_sync(0xffffffffu, wait(&bars.vfull[vent], (vuse / p.nv_entries) & 1));
      if (!ok) break;
      uint8_t* vrow = sV + vent * VB * kSlotBytes + r * 128;
      if constexpr (MASS)
        *reinterpret_cast<__half*>(vrow + KB * kSlotBytes + (sw << 4)) = __float2half_rn(f);
      const uint64_t f2 = f2_pack(f, f);
      // (rolled loops: the converters' code stays small beside the unrolled softmax loop that
      // shares each sub-partition's instruction cache; unrolled, the kernel took 2.23 vs 2.09 ms)
#pragma unroll 1
      for (int kb = 0; kb < KB; ++kb) {
#pragma unroll 1
        for (int h4 = 0; h4 < 8; h4 += 4) {
          uint4 w[4];
#pragma unroll
          for (int u = 0; u < 4; ++u)
            w[u] = *reinterpret_cast<const uint4*>(vrow + kb * kSlotBytes + (((h4 + u) ^ sw) << 4));
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            if (valid) {
              w[u].x = scale_bf16x2_to_f16x2_rn(w[u].x, f2);
              w[u].y = scale_bf16x2_to_f16x2_rn(w[u].y, f2);
              w[u].z = scale_bf16x2_to_f16x2_rn(w[u].z, f2);
              w[u].w = scale_bf16x2_to_f16x2_rn(w[u].w, f2);
            } else {
              w[u] = make_uint4(0, 0, 0, 0);  // padding rows: zeros, whatever they held
            }
            *reinterpret_cast<uint4*>(vrow + kb * kSlotBytes + (((h4 + u) ^ sw) << 4)) = w[u];
          }
        }
      }
      fence_async_shared();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.vconv[vent]);
      vent = (vent + 1 == p.nv_entries) ? 0 : vent + 1;
      ++vuse;
      tile_next(p, t);
    }
  } else {
    setmaxnreg_inc<kSoftmaxRegs>();
    // ------------------------------------------------------------ softmax warpgroups
    const int g = (warp - 8) >> 2;          // warpgroup: columns [g*NCOL, (g+1)*NCOL)
    const int q4 = warp & 3;                // TMEM lane quarter
    const int r = q4 * 32 + lane;           // token row of this thread
    const int col0 = g * NCOL;
    const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
    const float c2 = p.scale_log2;
    const uint64_t c2x2 = f2_pack(c2, c2);
    TilePos t;
    if (ntiles > 0) tile_seek(p, g0, t);
    int nseg = 0;
    int sl = 0, nmc = 0;  // tile index inside the segment's part, mass chains read
    bool ok = true;
    const uint32_t xbase = smem_u32(sX);
    int cur_b = -1, used = 0;
    if constexpr (MASS) {
      if (q4 == 0 && lane == 0)
        for (int c = 0; c < NCOL; ++c) sMass[col0 + c] = 0.f;
    }
    for (int i = 0; i < ntiles && ok; ++i) {
      if (t.b != cur_b) {
        cur_b = t.b;
        used = user_used(p, t.b);
      }
      const bool valid = r < used - t.j * kTileTokens;
      const bool first = (t.j == 0) || (i == 0);
      const bool last = (t.j == t.nb - 1) || (i == ntiles - 1);
      const int par = i & 1;
      sl = first ? 0 : sl + 1;

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

      // Row max over this warpgroup's columns (log2 units), then over the CTA's through the
      // other warpgroup's entry for the same row.
      float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
#pragma unroll
      for (int c = 0; c < NCOL; c += 8) {
        mx0 = max3f(mx0, __uint_as_float(sv[c + 0]), __uint_as_float(sv[c + 1]));
        mx1 = max3f(mx1, __uint_as_float(sv[c + 2]), __uint_as_float(sv[c + 3]));
        mx2 = max3f(mx2, __uint_as_float(sv[c + 4]), __uint_as_float(sv[c + 5]));
        mx3 = max3f(mx3, __uint_as_float(sv[c + 6]), __uint_as_float(sv[c + 7]));
      }
      const float mloc = valid ? fmaxf(max3f(mx0, mx1, mx2), mx3) * c2 : 0.f;
      sM[(par * 2 + g) * 128 + r] = mloc;
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.mxbar[par]);
      ok = __all_sync(0xffffffffu, wait(&bars.mxbar[par], (i >> 1) & 1));
      if (!ok) break;
      const float m = fmaxf(mloc, sM[(par * 2 + (g ^ 1)) * 128 + r]);

      // E = 2^(s c2 - m) as fp16 pairs, packed in place (word c / 2 holds columns c, c + 1),
      // and its fp32 row sum.
      const uint64_t negm = f2_pack(-m, -m);
      uint64_t acc0 = f2_pack(0.f, 0.f), acc1 = acc0;
#pragma unroll
      for (int c = 0; c < NCOL; c += 4) {
        float x0, x1, x2, x3;
        f2_unpack(f2_fma(f2_pack(__uint_as_float(sv[c]), __uint_as_float(sv[c + 1])), c2x2, negm), x0, x1);
        f2_unpack(f2_fma(f2_pack(__uint_as_float(sv[c + 2]), __uint_as_float(sv[c + 3])), c2x2, negm), x2, x3);
        const float e0 = ex2_approx(x0), e1 = ex2_approx(x1), e2 = ex2_approx(x2), e3 = ex2_approx(x3);
        acc0 = f2_add(acc0, f2_pack(e0, e1));
        acc1 = f2_add(acc1, f2_pack(e2, e3));
        sv[c / 2] = pack_f16x2(e0, e1);
        sv[c / 2 + 1] = pack_f16x2(e2, e3);
      }
      float a0, a1, b0, b1;
      f2_unpack(acc0, a0, a1);
      f2_unpack(acc1, b0, b1);
      const float lsum = valid ? (a0 + a1) + (b0 + b1) : 0.f;

      // (m, l) to every CTA of the cluster: asynchronous stores that count as transaction
      // bytes on the destination CTA's exchange barrier of this tile's slot.
      const int xs = i & (kXSlots - 1);
      const uint32_t xoff = static_cast<uint32_t>((((xs * CS + rank) * 2 + g) * 128 + r) * 8);
      const uint32_t xbar_local = smem_u32(&bars.xbar[xs]);
      for (int c = 0; c < CS; ++c)
        st_async_f32x2(mapa_shared(xbase + xoff, c), m, lsum, mapa_shared(xbar_local, c));

      // E into the swizzled MN-major B operand of MMA2, once MMA2 of the previous tile is done.
      if (i > 0) {
        ok = __all_sync(0xffffffffu, wait(&bars.pfree, (i - 1) & 1));
        if (!ok) break;
      }
#pragma unroll
      for (int c = 0; c < NCOL; c += 8) {
        const int jj = col0 + c;
        uint4 w = valid ? make_uint4(sv[c / 2], sv[c / 2 + 1], sv[c / 2 + 2], sv[c / 2 + 3]) : make_uint4(0, 0, 0, 0);
        uint8_t* dst = sP + (jj >> 6) * kSlotBytes + sw128_offset(r, (jj & 63) * 2);
        *reinterpret_cast<uint4*>(dst) = w;
      }
      fence_async_shared();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.pfull);

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
      if constexpr (MASS) {
        // End of a mass chain: row 0 of the M = 64 accumulator (TMEM lane 0) is added into the
        // segment's fp32 sums by lane 0 of the lane-quarter-0 warps; at the segment's end the
        // sums go to its partial slot.
        if (q4 == 0 && (last || (sl % kMassChain) == kMassChain - 1)) {
          ok = __all_sync(0xffffffffu, wait(&bars.mfull, nmc & 1));
          if (!ok) break;
          ++nmc;
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < NCOL; c += 8) {
            float mv[8];
            tmem_ld8(tMs + col0 + c, reinterpret_cast<uint32_t*>(mv));
            tmem_ld_wait();
            if (lane == 0) {
#pragma unroll
              for (int u = 0; u < 8; ++u) sMass[col0 + c + u] += mv[u];
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(&bars.mfree);
            if (last) {
              float* dst = p.mass_partial + static_cast<int64_t>((t.b * p.H + t.h) + cid) * p.k + rank * KC + col0;
              for (int c = 0; c < NCOL; ++c) {
                dst[c] = sMass[col0 + c];
                sMass[col0 + c] = 0.f;
              }
            }
          }
          __syncwarp();
        }
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

template <int D, int KC, bool MASS>
cudaError_t prepare_t(const ProtoFwdLaunch& L) {
  auto kern = sa_proto_fwd_kernel<D, KC, MASS>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.smem_bytes);
  if (e != cudaSuccess) return e;
  if (L.cluster > 1) e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  return e;
}

// Clusters of this configuration that the device holds at once (0 if the query fails).
template <int D, int KC, bool MASS>
int max_clusters_t(const ProtoFwdLaunch& L) {
  if (prepare_t<D, KC, MASS>(L) != cudaSuccess) return 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(L.num_clusters * L.cluster, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = L.smem_bytes;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = L.cluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, sa_proto_fwd_kernel<D, KC, MASS>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

template <int D, int KC, bool MASS>
cudaError_t launch_t(const ProtoFwdLaunch& L, const CUtensorMap& mQ, const CUtensorMap& mK,
                     const CUtensorMap& mV, const ProtoFwdParams& p, cudaStream_t stream) {
  auto kern = sa_proto_fwd_kernel<D, KC, MASS>;
  cudaError_t e = prepare_t<D, KC, MASS>(L);
  if (e != cudaSuccess) return e;
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

constexpr size_t kSmemBudget = 227 * 1024;

}  // namespace

bool proto_fwd_plan(int D, int k, int num_sms, bool mass, ProtoFwdLaunch* out, int* nk_slots, int* nv_entries) {
  if (D != 64 && D != 128) return false;
  if (k < 16 || k % 16 != 0) return false;
  const int per_cta = mass ? 128 : kMaxProtosPerCta;  // the mass accumulator needs TMEM columns
  const int cs = (k + per_cta - 1) / per_cta;
  if (cs > 8 || k % cs != 0) return false;
  const int kc = k / cs;
  if (kc % 16 != 0) return false;
  if (!(kc == 16 || kc == 32 || kc == 64 || kc == 96 || kc == 128 || kc == 192 || kc == 256)) return false;
  if (mass && kc > 128) return false;
  // Fill shared memory: prefer deep rings for K (16 KB slots) and V (tile entries).
  const int kb = D / 64;
  int best_nk = 0, best_nv = 0;
  for (int nv = 1; nv <= kMaxRing; ++nv) {
    for (int nk = kb; nk <= kMaxRing; ++nk) {
      SmemLayout L = smem_layout(D, kc, cs, nk, nv, mass);
      if (L.total > kSmemBudget) continue;
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
  out->mass = mass;
  out->smem_bytes = smem_layout(D, kc, cs, best_nk, best_nv, mass).total;
  *nk_slots = best_nk;
  *nv_entries = best_nv;
  return true;
}

#define SKA_PROTO_TABLE(X)                                                                                   \
  X(64, 16, false) X(64, 32, false) X(64, 64, false) X(64, 96, false) X(64, 128, false) X(64, 192, false)   \
  X(64, 256, false) X(128, 16, false) X(128, 32, false) X(128, 64, false) X(128, 96, false)                 \
  X(128, 128, false) X(128, 192, false) X(128, 256, false) X(64, 16, true) X(64, 32, true) X(64, 64, true)  \
  X(64, 96, true) X(64, 128, true) X(128, 16, true) X(128, 32, true) X(128, 64, true) X(128, 96, true)      \
  X(128, 128, true)

int proto_fwd_max_clusters(int D, const ProtoFwdLaunch& L) {
  // one query per (device, configuration): the answer does not change while the process lives
  struct Entry { int dev, D, kc, cs, mass, n; };
  static Entry cache[64];
  static int used = 0;
  static std::mutex mu;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < used; ++i)
    if (cache[i].dev == dev && cache[i].D == D && cache[i].kc == L.kc && cache[i].cs == L.cluster &&
        cache[i].mass == int(L.mass))
      return cache[i].n;
  int n = 0;
#define SKA_PROTO_Q(DD, KK, MM) \
  if (D == DD && L.kc == KK && L.mass == MM) n = max_clusters_t<DD, KK, MM>(L);
  SKA_PROTO_TABLE(SKA_PROTO_Q)
#undef SKA_PROTO_Q
  if (used < 64) cache[used++] = Entry{dev, D, L.kc, L.cluster, int(L.mass), n};
  return n;
}

cudaError_t launch_proto_fwd(int D, const ProtoFwdLaunch& L, const CUtensorMap& mQ, const CUtensorMap& mK,
                             const CUtensorMap& mV, const ProtoFwdParams& p, cudaStream_t stream) {
#define SKA_PROTO_CASE(DD, KK, MM) \
  if (D == DD && L.kc == KK && L.mass == MM) return launch_t<DD, KK, MM>(L, mQ, mK, mV, p, stream);
  SKA_PROTO_TABLE(SKA_PROTO_CASE)
#undef SKA_PROTO_CASE
  return cudaErrorInvalidValue;
}

}  // namespace ska
