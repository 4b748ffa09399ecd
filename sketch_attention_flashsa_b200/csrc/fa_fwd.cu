// Row-softmax forward on sm_100a, shared by two operations:
//
// * Token-wise SA: the "vanilla attention" normalisation that SequenceO1 §5.1 / Table 1
//   compares with the paper's prototype-wise Eq. (8): every prototype j takes a softmax over
//   the valid history tokens of its user, sketch_j = sum_i softmax_i(scale q_j . k_i) v_i.
// * STCA (§2.3, applied in §3.4 to the recent suffix and to the sketch, many targets of one
//   user batched by MRLB, §4.2): out_t = softmax(scale q_t K^T) V over the keys
//   [suffix rows of the user (the first target_kv_len[t] of them) ; the user's sketch rows].
//
// A "stream" is one 128-row query tile of one (user, head): prototypes for SA, targets for
// STCA. Streams are walked in 128-key tiles with an online (running max / running sum)
// softmax; the key tiles of all streams are concatenated and split evenly across persistent
// CTAs, each CTA writes an unnormalised partial (O, max, sum) per stream it touches, and a
// combine kernel merges the partials of a stream by their log-sum-exp weights.
//
// Per key tile, one CTA (384 threads) holds two query tiles Q_0, Q_1 (query tiles 2u, 2u+1 of a
// stream pair) and, for w = 0, 1:
//   MMA1  S_w = Q_w . K_tile^T        M=128, N=128, K=d   -> TMEM columns [128 w, 128 w + 128)
//   softmax warpgroup w (thread = query row of Q_w): mask, running max (O_w rescaled in TMEM only
//         when the max grows by more than 2^8), P_w = 2^(s c - m) as bf16 pairs written back over
//         the first 64 columns of S_w
//   MMA2  O_w += P_w . V_tile         M=128, N=d, K=128 keys, A read from TMEM  -> TMEM
// The MMA issuer orders MMA2(P_w, tile) before MMA1(Q_w, next tile) into the same columns, and
// tcgen05 MMAs of one thread run in issue order, so S_w is only overwritten once P_w has been
// read. The two warpgroups settle half a tile apart: while one computes its exponentials, the
// tensor core runs the other's two MMAs.
// Warp 0: TMA producer of Q and K; warp 1: TMEM owner + MMA issuer; warp 2: TMA producer of V;
// warps 4-7 and 8-11: softmax warpgroups 0 and 1.
#include <algorithm>
#include <cmath>

#include "ska_internal.h"
#include "ska_ptx.cuh"

namespace ska {

namespace {

constexpr int kFaThreads = 384;
// Registers per thread after the split: the launch gives every thread 168 (three warps per
// sub-partition); warpgroup 0 drops to 96 and the two softmax warpgroups rise to 200
// (96 x 128 + 200 x 256 <= 168 x 384, and 32 x (96 + 2 x 200) registers per sub-partition fit in
// its 16,384). With this split neither instantiation spills; with 168 for all they spill 72-88 bytes.
constexpr uint32_t kFaRoleRegs = 96;
constexpr uint32_t kFaSoftmaxRegs = 200;
constexpr int kFaSlot = 16384;         // one [128 rows x 64 bf16] swizzled block
constexpr int kFaMaxRing = 8;
constexpr float kRescaleThreshold = 8.f;  // log2 units

__host__ __device__ constexpr int fa_q_bytes(int D) { return 128 * D * 2; }

struct FaLayout {
  uint32_t q_off, k_off, v_off, total;
};

__host__ __device__ inline FaLayout fa_layout(int D, int nk, int nv) {
  FaLayout L;
  uint32_t off = 0;
  L.q_off = off;
  off += 2 * fa_q_bytes(D);           // Q_0, Q_1
  L.k_off = off;
  off += nk * (D / 64) * kFaSlot;     // K ring: tile entries
  L.v_off = off;
  off += nv * (D / 64) * kFaSlot;     // V ring: tile entries
  L.total = off;
  return L;
}

// ---------------------------------------------------------------- per-user geometry
__device__ __forceinline__ int fa_used(const FaFwdParams& p, int b) {
  int len = p.cu_keys[b + 1] - p.cu_keys[b];
  if (p.seqused) len = min(len, p.seqused[b]);
  return max(len, 0);
}

// query tiles of user b
__device__ __forceinline__ int fa_qtiles(const FaFwdParams& p, int b) {
  if (p.mode == 0) return (p.k + 127) / 128;
  return (max(p.cu_q[b + 1] - p.cu_q[b], 0) + 127) / 128;
}

// key tiles of user b: [history or suffix tiles ; sketch tiles (STCA)]
__device__ __forceinline__ int fa_hist_tiles(const FaFwdParams& p, int b) { return (fa_used(p, b) + 127) / 128; }
__device__ __forceinline__ int fa_ktiles(const FaFwdParams& p, int b) {
  return fa_hist_tiles(p, b) + (p.mode == 1 ? (p.ks + 127) / 128 : 0);
}

// Work layout. Columns are the key tiles of every (user, head): user b contributes H * n_b
// columns (n_b key tiles per head), in order (b, h, j). G is the largest number of 128-row
// query tiles of any user; persistent CTAs form groups of (G + 1) / 2, and the CTAs of group g
// walk the same contiguous column range together, CTA (g, u) with query tiles 2u and 2u + 1, so
// a K/V tile is read from DRAM once and from L2 by the other CTAs of the group. Columns of users
// with fewer than 2u + 1 query tiles are skipped by that CTA; a user with exactly 2u + 1 leaves
// its second query tile (and second softmax warpgroup) idle.
struct FaPos {
  int b, h, j;   // user, head, key tile
  int nb, qtn;   // key tiles per head of user b, query tiles of user b
};

__device__ __forceinline__ void fa_user(const FaFwdParams& p, FaPos& t) {
  t.nb = fa_ktiles(p, t.b);
  t.qtn = fa_qtiles(p, t.b);
}

// First processable column at or after column g for query tile qt (t.b == B when none).
__device__ __forceinline__ void fa_seek(const FaFwdParams& p, int g, int qt, FaPos& t) {
  int lo = 0, hi = p.B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.tile_prefix[mid] <= g) lo = mid; else hi = mid - 1;
  }
  t.b = lo;
  fa_user(p, t);
  const int off = g - p.tile_prefix[lo];
  if (t.nb > 0 && off < p.H * t.nb) {
    t.h = off / t.nb;
    t.j = off - t.h * t.nb;
  } else {
    t.h = p.H;  // past this user
    t.j = 0;
  }
  if (qt >= t.qtn || t.h >= p.H) {
    t.h = 0;
    t.j = 0;
    do {
      ++t.b;
      if (t.b >= p.B) return;
      fa_user(p, t);
    } while (t.nb == 0 || qt >= t.qtn);
  }
}

__device__ __forceinline__ void fa_next(const FaFwdParams& p, int qt, FaPos& t) {
  if (++t.j < t.nb) return;
  t.j = 0;
  if (++t.h < p.H) return;
  t.h = 0;
  do {
    ++t.b;
    if (t.b >= p.B) return;
    fa_user(p, t);
  } while (t.nb == 0 || qt >= t.qtn);
}

// Column index of a position.
__device__ __forceinline__ int fa_col(const FaFwdParams& p, const FaPos& t) {
  return p.tile_prefix[t.b] + t.h * t.nb + t.j;
}

// Number of columns in [c0, c1) that query tile qt processes.
__device__ __forceinline__ int fa_count(const FaFwdParams& p, int qt, int c0, int c1) {
  int n = 0;
  int lo = 0, hi = p.B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.tile_prefix[mid] <= c0) lo = mid; else hi = mid - 1;
  }
  for (int b = lo; b < p.B; ++b) {
    const int u0 = p.tile_prefix[b], u1 = p.tile_prefix[b + 1];
    if (u0 >= c1) break;
    if (qt < fa_qtiles(p, b)) n += max(0, min(u1, c1) - max(u0, c0));
  }
  return n;
}

// ---------------------------------------------------------------- schedule
// One block: tile_prefix[b] = sum_{b' < b} H * n_b'; columns per group; the largest number of
// query tiles of any user (a device-side error when it exceeds the group size G); clears status.
__global__ void __launch_bounds__(1024) fa_schedule_kernel(const FaFwdParams p, int num_groups, int G) {
  __shared__ long long part_t[1024];
  __shared__ int part_q[1024];
  const int t = threadIdx.x;
  const int per = (p.B + 1023) / 1024;
  const int lo = min(p.B, t * per), hi = min(p.B, lo + per);
  long long st = 0;
  int qmax = 0;
  for (int b = lo; b < hi; ++b) {
    st += static_cast<long long>(p.H) * fa_ktiles(p, b);
    qmax = max(qmax, fa_qtiles(p, b));
  }
  part_t[t] = st;
  part_q[t] = qmax;
  __syncthreads();
  for (int off = 1; off < 1024; off <<= 1) {
    const long long vt = (t >= off) ? part_t[t - off] : 0;
    const int vq = (t >= off) ? part_q[t - off] : 0;
    __syncthreads();
    part_t[t] += vt;
    part_q[t] = max(part_q[t], vq);
    __syncthreads();
  }
  long long rt = (t == 0) ? 0 : part_t[t - 1];
  for (int b = lo; b < hi; ++b) {
    const_cast<int32_t*>(p.tile_prefix)[b] = static_cast<int32_t>(rt);
    rt += static_cast<long long>(p.H) * fa_ktiles(p, b);
  }
  if (t == 1023) {
    const_cast<int32_t*>(p.tile_prefix)[p.B] = static_cast<int32_t>(part_t[1023]);
    const int total = static_cast<int>(part_t[1023]);
    p.hdr->total_tiles = total;
    p.hdr->tiles_per_cluster = (total + num_groups - 1) / num_groups;
    p.hdr->status = (part_q[1023] > G) ? static_cast<int>(SKA_ERR_INVALID_VALUE) : 0;
  }
}

// ---------------------------------------------------------------- combine
// One block per (user, head, query tile) up to B * H * G; thread r merges row r of the stream
// over the partial slots ((b H + h) + g) G + qt of the groups g that walked its columns. When an
// earlier kernel of the call recorded an error (a bounded wait that ran out, a user with more
// targets than max_targets) every output of the call is NaN. Token-wise SA also writes the
// mass of each prototype, sum_i A[j, i], which the softmax over tokens makes 1 (0 for a user
// without valid tokens).
__global__ void __launch_bounds__(128) fa_combine_kernel(const FaFwdParams p, int D, int G, float* __restrict__ out,
                                                         float* __restrict__ lse, float* __restrict__ mass) {
  const bool failed = *reinterpret_cast<const volatile int32_t*>(&p.hdr->status) != 0;
  const int qt = blockIdx.x % G;
  const int bh = blockIdx.x / G;
  const int b = bh / p.H, h = bh - b * p.H;
  if (b >= p.B) return;
  if (qt >= fa_qtiles(p, b)) return;
  const int nb = fa_ktiles(p, b);
  const int W = p.hdr->tiles_per_cluster;
  int g0 = 0, g1 = -1;
  if (nb > 0 && W > 0) {
    const int c0 = p.tile_prefix[b] + h * nb;
    g0 = c0 / W;
    g1 = (c0 + nb - 1) / W;
  }
  const int r = threadIdx.x;
  const int nq = (p.mode == 0) ? p.k : (p.cu_q[b + 1] - p.cu_q[b]);
  auto slot = [&](int g, int q) { return (static_cast<int64_t>(bh + g) * G + qt) * 128 + (q & 127); };
  // Rows qt*128 + r, then G*128 further on: the second and later rows exist only when a user has
  // more query tiles than G, which the schedule records as an error; they are written as NaN.
  for (int q = qt * 128 + r; q < nq; q += G * 128) {
    const bool bad = failed || q >= G * 128;
    float M = -INFINITY;
    float L = 0.f;
    if (!bad) {
      for (int g = g0; g <= g1; ++g) M = fmaxf(M, p.part_ml[slot(g, q) * 2]);
      for (int g = g0; g <= g1; ++g) {
        const float mg = p.part_ml[slot(g, q) * 2];
        if (mg != -INFINITY) L += p.part_ml[slot(g, q) * 2 + 1] * exp2f(mg - M);
      }
    }
    const float inv = (L > 0.f) ? 1.f / L : 0.f;
    int64_t orow;
    if (p.mode == 0) orow = (static_cast<int64_t>(b) * p.H + h) * p.k + q;
    else orow = static_cast<int64_t>(p.cu_q[b] + q) * p.H + h;
    float* dst = out + orow * D;
    for (int dd = 0; dd < D; dd += 4) {
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      if (!bad) {
        for (int g = g0; g <= g1; ++g) {
          const float mg = p.part_ml[slot(g, q) * 2];
          if (mg == -INFINITY) continue;
          const float wg = exp2f(mg - M);
          const float4 v = *reinterpret_cast<const float4*>(p.part_o + slot(g, q) * D + dd);
          acc.x += wg * v.x; acc.y += wg * v.y; acc.z += wg * v.z; acc.w += wg * v.w;
        }
        acc.x *= inv; acc.y *= inv; acc.z *= inv; acc.w *= inv;
      } else {
        acc = make_float4(NAN, NAN, NAN, NAN);
      }
      *reinterpret_cast<float4*>(dst + dd) = acc;
    }
    if (lse) lse[orow] = bad ? NAN : (L > 0.f) ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
    if (mass) mass[orow] = bad ? NAN : (L > 0.f) ? 1.f : 0.f;
  }
}

struct FaBars {
  uint64_t kfull[kFaMaxRing], kempty[kFaMaxRing], vfull[kFaMaxRing], vempty[kFaMaxRing];
  uint64_t qfull, qfree, sfull[2], pfull[2], ofull[2], ofree[2], drain;
  uint32_t tmem_base;
  int abort_flag;
};

struct FaWaiter {
  FaBars* bars;
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

// Q tile row (in the Q map) and column base for query tile qt of the stream at t.
__device__ __forceinline__ void fa_q_coord(const FaFwdParams& p, const FaPos& t, int qt, int D, int& c0,
                                           int& row) {
  const int h = t.h;
  if (p.mode == 0) {
    c0 = 0;
    row = (p.q_per_user ? t.b * p.H * p.k : 0) + h * p.k + qt * 128;
  } else {
    c0 = h * D;
    row = p.cu_q[t.b] + qt * 128;
  }
}

// K / V tile coordinates of the key tile at t: [history or suffix rows ; sketch rows (STCA)].
__device__ __forceinline__ bool fa_kv_coord(const FaFwdParams& p, const FaPos& t, int D, int& c0, int& row) {
  const int nh = fa_hist_tiles(p, t.b);
  if (t.j < nh) {
    c0 = t.h * D;
    row = p.cu_keys[t.b] + t.j * 128;
    return false;
  }
  c0 = 0;
  row = (t.b * p.H + t.h) * p.ks + (t.j - nh) * 128;
  return true;
}

// Waits of the producers at exit for their loads still in flight (none may land after exit).
__device__ __forceinline__ void fa_drain_ring(FaWaiter& wait, uint64_t* full, int slots, int uses) {
  for (int e = 0; e < slots; ++e) {
    const int fills = (uses > e) ? (uses - e - 1) / slots + 1 : 0;
    if (fills > 0) wait(&full[e], (fills - 1) & 1, true);
  }
}

template <int D>
__global__ void __launch_bounds__(kFaThreads, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapK,
                  const __grid_constant__ CUtensorMap mapV, const __grid_constant__ CUtensorMap mapKs,
                  const __grid_constant__ CUtensorMap mapVs, const FaFwdParams p) {
  constexpr int KB = D / 64;
  constexpr int kTileBytes = KB * kFaSlot;
  constexpr int kQBytes = fa_q_bytes(D);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ FaBars bars;
  const FaLayout L = fa_layout(D, p.nk_slots, p.nv_entries);
  uint8_t* sQ = smem + L.q_off;
  uint8_t* sK = smem + L.k_off;
  uint8_t* sV = smem + L.v_off;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int nk = p.nk_slots, nv = p.nv_entries;

  if (threadIdx.x == 0) {
    for (int i = 0; i < nk; ++i) { mbar_init(&bars.kfull[i], 1); mbar_init(&bars.kempty[i], 1); }
    for (int i = 0; i < nv; ++i) { mbar_init(&bars.vfull[i], 1); mbar_init(&bars.vempty[i], 1); }
    mbar_init(&bars.qfull, 1);
    mbar_init(&bars.qfree, 1);
    for (int w = 0; w < 2; ++w) {
      mbar_init(&bars.sfull[w], 1);
      mbar_init(&bars.pfull[w], 4);  // the four warps of softmax warpgroup w
      mbar_init(&bars.ofull[w], 1);
      mbar_init(&bars.ofree[w], 4);
    }
    mbar_init(&bars.drain, 1);
    bars.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // TMEM columns: S_0 [0, 128), S_1 [128, 256), O_0 [256, 256 + D), O_1 [256 + D, 256 + 2 D)
  const uint32_t tbase = bars.tmem_base;
  FaWaiter wait{&bars, &p.hdr->status, p.budget_ns};
  // group of (G + 1) / 2 CTAs walking one column range; this CTA's query tiles qt0, qt0 + 1
  const int G = p.group;
  const int Gc = (G + 1) >> 1;
  const int grp = blockIdx.x / Gc;
  const int qt0 = 2 * (blockIdx.x % Gc);
  const int ngroups = gridDim.x / Gc;
  const int total = p.hdr->total_tiles;
  const int W = p.hdr->tiles_per_cluster;
  const int c0 = grp * W, c1 = min(total, c0 + W);
  const int ntiles = (grp < ngroups && W > 0 && c0 < total && p.hdr->status == 0) ? fa_count(p, qt0, c0, c1) : 0;

  if (warp < 4) {
    // warps 0-3 (producers, MMA issuer, one idle warp) give registers to the softmax warpgroups
    setmaxnreg_dec<kFaRoleRegs>();
    if (warp == 0) {
      // ------------------------------------------------------------ TMA producer: Q pairs and K
      if (lane == 0 && ntiles > 0) {
        FaPos t;
        fa_seek(p, c0, qt0, t);
        int kent = 0, kuse = 0, nq = 0;
        bool ok = true;
        bool skip_first = (p.debug_flags & 1u) != 0;
        for (int i = 0; i < ntiles && ok; ++i) {
          if (t.j == 0 || i == 0) {
            // the stream's query tiles, once the previous stream's last MMA1 has read sQ
            if (nq > 0) ok = wait(&bars.qfree, (nq - 1) & 1);
            if (!ok) break;
            const int nqt = (qt0 + 1 < t.qtn) ? 2 : 1;
            int qc0, qrow;
            fa_q_coord(p, t, qt0, D, qc0, qrow);
            mbar_expect_tx(&bars.qfull, kQBytes * nqt);
            for (int w = 0; w < nqt; ++w)
              for (int kb = 0; kb < KB; ++kb)
                tma_load_2d(sQ + w * kQBytes + kb * kFaSlot, &mapQ, &bars.qfull, qc0 + kb * 64, qrow + w * 128);
            ++nq;
          }
          ok = wait(&bars.kempty[kent], ((kuse / nk) & 1) ^ 1);
          if (!ok) break;
          int kc0, krow;
          const CUtensorMap* mk = fa_kv_coord(p, t, D, kc0, krow) ? &mapKs : &mapK;
          if (skip_first) {
            skip_first = false;  // withhold this arrival: the MMA warp's wait must run out
          } else {
            mbar_expect_tx(&bars.kfull[kent], kTileBytes);
            for (int kb = 0; kb < KB; ++kb)
              tma_load_2d(sK + kent * kTileBytes + kb * kFaSlot, mk, &bars.kfull[kent], kc0 + kb * 64, krow);
          }
          kent = (kent + 1 == nk) ? 0 : kent + 1;
          ++kuse;
          fa_next(p, qt0, t);
        }
        fa_drain_ring(wait, bars.kfull, nk, kuse);
        if (nq > 0) wait(&bars.qfull, (nq - 1) & 1, true);
      }
    } else if (warp == 2) {
      // ------------------------------------------------------------ TMA producer: V
      if (lane == 0 && ntiles > 0) {
        FaPos t;
        fa_seek(p, c0, qt0, t);
        int vent = 0, vuse = 0;
        bool ok = true;
        for (int i = 0; i < ntiles && ok; ++i) {
          ok = wait(&bars.vempty[vent], ((vuse / nv) & 1) ^ 1);
          if (!ok) break;
          int vc0, vrow;
          const CUtensorMap* mv = fa_kv_coord(p, t, D, vc0, vrow) ? &mapVs : &mapV;
          mbar_expect_tx(&bars.vfull[vent], kTileBytes);
          for (int kb = 0; kb < KB; ++kb)
            tma_load_2d(sV + vent * kTileBytes + kb * kFaSlot, mv, &bars.vfull[vent], vc0 + kb * 64, vrow);
          vent = (vent + 1 == nv) ? 0 : vent + 1;
          ++vuse;
          fa_next(p, qt0, t);
        }
        fa_drain_ring(wait, bars.vfull, nv, vuse);
      }
    } else if (warp == 1) {
      // ------------------------------------------------------------ MMA issuer
      // Order per key tile i: for w = 0, 1: MMA2(P_w, V_i) -> O_w, then MMA1(Q_w, K_{i+1}) -> S_w.
      if (lane == 0 && ntiles > 0) {
        constexpr uint32_t idesc1 = idesc_bf16_f32(128, 128, false, false);
        constexpr uint32_t idesc2 = idesc_bf16_f32(128, D, false, true);
        auto mma1 = [&](int w, uint32_t kbase) {
          const uint32_t qbase = smem_u32(sQ + w * kQBytes);
  #pragma unroll
          for (int s = 0; s < D / 16; ++s) {
            const uint64_t ad = sw128_desc(qbase + (s / 4) * kFaSlot + (s % 4) * 32, 16, 1024);
            const uint64_t bd = sw128_desc(kbase + (s / 4) * kFaSlot + (s % 4) * 32, 16, 1024);
            umma_bf16(tbase + w * 128, ad, bd, idesc1, s > 0 ? 1u : 0u);
          }
          umma_commit(&bars.sfull[w]);
        };
        auto mma2 = [&](int w, uint32_t vbase, bool fresh) {
  #pragma unroll
          for (int s = 0; s < 8; ++s) {
            const uint64_t bd = sw128_desc(vbase + s * 2048, kFaSlot, 1024);
            umma_bf16_ts(tbase + 256 + w * D, tbase + w * 128 + s * 8, bd, idesc2, (fresh && s == 0) ? 0u : 1u);
          }
        };
        FaPos t;
        fa_seek(p, c0, qt0, t);
        int kent = 0, kuse = 0, vent = 0, vuse = 0, nq = 0;
        int np[2] = {0, 0}, nseg[2] = {0, 0};
        bool ok = true;
        {
          // MMA1 of the first tile
          ok = wait(&bars.qfull, 0) && wait(&bars.kfull[0], 0);
          if (ok) {
            ++nq;
            tc_fence_after();
            const uint32_t kbase = smem_u32(sK);
            mma1(0, kbase);
            if (qt0 + 1 < t.qtn) mma1(1, kbase);
            umma_commit(&bars.kempty[0]);
            if (t.j == t.nb - 1 || ntiles == 1) umma_commit(&bars.qfree);
            kent = (nk == 1) ? 0 : 1;
            ++kuse;
          }
        }
        for (int i = 0; i < ntiles && ok; ++i) {
          const bool first = (t.j == 0) || (i == 0);
          const bool last = (t.j == t.nb - 1) || (i == ntiles - 1);
          const bool q1 = qt0 + 1 < t.qtn;
          const bool more = i + 1 < ntiles;
          FaPos tn = t;
          if (more) fa_next(p, qt0, tn);
          const bool nq1 = more && (qt0 + 1 < tn.qtn);
          const bool nfirst = more && (tn.j == 0);
          const bool nlast = more && ((tn.j == tn.nb - 1) || (i + 1 == ntiles - 1));
          ok = wait(&bars.vfull[vent], (vuse / nv) & 1);
          if (!ok) break;
          const uint32_t vbase = smem_u32(sV + vent * kTileBytes);
          const uint32_t knext = smem_u32(sK + kent * kTileBytes);
          bool next_in = false;
          // Q (first tile of a stream) and K of tile i + 1 resident
          auto next_ready = [&]() -> bool {
            if (next_in) return true;
            if (nfirst) {
              if (!wait(&bars.qfull, nq & 1)) return false;
              ++nq;
            }
            if (!wait(&bars.kfull[kent], (kuse / nk) & 1)) return false;
            next_in = true;
            return true;
          };
  #pragma unroll
          for (int w = 0; w < 2; ++w) {
            if (w == 1 && !q1) break;
            ok = wait(&bars.pfull[w], np[w] & 1);
            if (!ok) break;
            ++np[w];
            if (first && nseg[w] > 0) {
              ok = wait(&bars.ofree[w], (nseg[w] - 1) & 1);
              if (!ok) break;
            }
            tc_fence_after();
            mma2(w, vbase, first);
            if (last) {
              umma_commit(&bars.ofull[w]);
              ++nseg[w];
            }
            if (more && (w == 0 || nq1)) {
              ok = next_ready();
              if (!ok) break;
              tc_fence_after();
              mma1(w, knext);
            }
          }
          if (!ok) break;
          if (nq1 && !q1) {
            // a stream with two query tiles after one with a single tile
            ok = next_ready();
            if (!ok) break;
            tc_fence_after();
            mma1(1, knext);
          }
          umma_commit(&bars.vempty[vent]);
          vent = (vent + 1 == nv) ? 0 : vent + 1;
          ++vuse;
          if (more) {
            umma_commit(&bars.kempty[kent]);
            if (nlast) umma_commit(&bars.qfree);
            kent = (kent + 1 == nk) ? 0 : kent + 1;
            ++kuse;
          }
          t = tn;
        }
        umma_commit(&bars.drain);
        wait(&bars.drain, 0, true);
      }
    }
  } else {
    setmaxnreg_inc<kFaSoftmaxRegs>();
    // ------------------------------------------------------------ softmax warpgroups
    // Warpgroup w (warps 4-7, 8-11) owns query tile qt0 + w: thread r holds query row r, its
    // running maximum m (the reference P is scaled against) and its running sum l.
    const int w = (warp - 4) >> 2;
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
    const uint32_t tS = tbase + w * 128 + lane_off;
    const uint32_t tO = tbase + 256 + w * D + lane_off;
    const float c2 = p.scale_log2;
    const uint64_t c2x2 = f2_pack(c2, c2);
    FaPos t;
    if (ntiles > 0) fa_seek(p, c0, qt0, t);
    float m = -INFINITY, l = 0.f;
    int ns = 0, nseg = 0;
    bool ok = true;
    int nh = 0, hlen = 0;  // this stream's history tiles and this row's valid history keys
    for (int i = 0; i < ntiles && ok; ++i) {
      if (w == 0 || qt0 + 1 < t.qtn) {
        const bool first = (t.j == 0) || (i == 0);
        const bool last = (t.j == t.nb - 1) || (i == ntiles - 1);
        if (first) {
          m = -INFINITY;
          l = 0.f;
          // constant over the key tiles of a stream: read once
          hlen = fa_used(p, t.b);
          nh = (hlen + 127) / 128;
          if (p.mode == 1 && p.kv_len) {
            const int q = (qt0 + w) * 128 + r;
            const int nq = p.cu_q[t.b + 1] - p.cu_q[t.b];
            if (q < nq) hlen = min(hlen, max(p.kv_len[p.cu_q[t.b] + q], 0));
          }
        }
        // valid keys of this tile for this row
        const int nvalid = (t.j < nh) ? hlen - t.j * 128 : p.ks - (t.j - nh) * 128;

        ok = __all_sync(0xffffffffu, wait(&bars.sfull[w], ns & 1));
        if (!ok) break;
        ++ns;
        tc_fence_after();
        uint32_t sv[128];
#pragma unroll
        for (int c = 0; c < 128; c += 32) tmem_ld32(tS + c, sv + c);
        tmem_ld_wait();
        if (nvalid < 128) {
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c >= nvalid) sv[c] = __float_as_uint(-INFINITY);
        }
        float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
#pragma unroll
        for (int c = 0; c < 128; c += 8) {
          mx0 = max3f(mx0, __uint_as_float(sv[c + 0]), __uint_as_float(sv[c + 1]));
          mx1 = max3f(mx1, __uint_as_float(sv[c + 2]), __uint_as_float(sv[c + 3]));
          mx2 = max3f(mx2, __uint_as_float(sv[c + 4]), __uint_as_float(sv[c + 5]));
          mx3 = max3f(mx3, __uint_as_float(sv[c + 6]), __uint_as_float(sv[c + 7]));
        }
        const float mt = fmaxf(max3f(mx0, mx1, mx2), mx3) * c2;
        // lazy rescale: move the reference only when the max grows by more than 2^8
        float factor = 1.f;
        if (mt > m + kRescaleThreshold || (m == -INFINITY && mt > -INFINITY)) {
          factor = (m == -INFINITY) ? 0.f : ex2_approx(m - mt);
          m = mt;
        }
        const float mref = (m == -INFINITY) ? 0.f : m;
        const uint64_t negm = f2_pack(-mref, -mref);
        uint64_t acc0 = f2_pack(0.f, 0.f), acc1 = acc0;
        // P as bf16 pairs, packed in place: word c / 2 holds columns c, c + 1
#pragma unroll
        for (int c = 0; c < 128; c += 4) {
          float x0, x1, x2, x3;
          f2_unpack(f2_fma(f2_pack(__uint_as_float(sv[c]), __uint_as_float(sv[c + 1])), c2x2, negm), x0, x1);
          f2_unpack(f2_fma(f2_pack(__uint_as_float(sv[c + 2]), __uint_as_float(sv[c + 3])), c2x2, negm), x2, x3);
          const float e0 = ex2_approx(x0), e1 = ex2_approx(x1), e2 = ex2_approx(x2), e3 = ex2_approx(x3);
          acc0 = f2_add(acc0, f2_pack(e0, e1));
          acc1 = f2_add(acc1, f2_pack(e2, e3));
          sv[c / 2] = pack_bf16x2(e0, e1);
          sv[c / 2 + 1] = pack_bf16x2(e2, e3);
        }
        float a0, a1, b0, b1;
        f2_unpack(acc0, a0, a1);
        f2_unpack(acc1, b0, b1);
        l = l * factor + ((a0 + a1) + (b0 + b1));
        tmem_st32(tS, sv);
        tmem_st32(tS + 32, sv + 32);
        // O_w rows whose reference moved are rescaled in TMEM: MMA2 of this warpgroup's previous
        // tile completed before S_w was written (sfull)
        if (!first && __any_sync(0xffffffffu, factor != 1.f)) {
#pragma unroll 1
          for (int c = 0; c < D; c += 32) {
            uint32_t ov[32];
            tmem_ld32(tO + c, ov);
            tmem_ld_wait();
#pragma unroll
            for (int u = 0; u < 32; ++u) ov[u] = __float_as_uint(__uint_as_float(ov[u]) * factor);
            tmem_st32(tO + c, ov);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.pfull[w]);

        if (last) {
          ok = __all_sync(0xffffffffu, wait(&bars.ofull[w], nseg & 1));
          if (!ok) break;
          tc_fence_after();
          // slot of (column stream (b, h), group, query tile): unique along the column staircase
          const int slot = ((t.b * p.H + t.h) + grp) * G + qt0 + w;
          float* dst = p.part_o + (static_cast<int64_t>(slot) * 128 + r) * D;
#pragma unroll 1
          for (int c = 0; c < D; c += 32) {
            uint32_t ov[32];
            tmem_ld32(tO + c, ov);
            tmem_ld_wait();
#pragma unroll
            for (int u = 0; u < 32; u += 4)
              *reinterpret_cast<float4*>(dst + c + u) = make_float4(__uint_as_float(ov[u]), __uint_as_float(ov[u + 1]),
                                                                    __uint_as_float(ov[u + 2]), __uint_as_float(ov[u + 3]));
          }
          p.part_ml[(static_cast<int64_t>(slot) * 128 + r) * 2] = m;
          p.part_ml[(static_cast<int64_t>(slot) * 128 + r) * 2 + 1] = l;
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars.ofree[w]);
          ++nseg;
        }
      }
      fa_next(p, qt0, t);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

template <int D>
cudaError_t fa_launch_t(int num_ctas, size_t smem, const CUtensorMap& mQ, const CUtensorMap& mK,
                        const CUtensorMap& mV, const CUtensorMap& mKs, const CUtensorMap& mVs,
                        const FaFwdParams& p, cudaStream_t stream) {
  auto kern = fa_fwd_kernel<D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<num_ctas, kFaThreads, smem, stream>>>(mQ, mK, mV, mKs, mVs, p);
  return cudaGetLastError();
}

}  // namespace

bool fa_fwd_plan(int D, int num_sms, int* num_ctas, size_t* smem_bytes, int* nk, int* nv) {
  if (D != 64 && D != 128) return false;
  const size_t budget = 227 * 1024 - 1024 - 512;
  int best_k = 0, best_v = 0;
  for (int v = 1; v <= kFaMaxRing; ++v)
    for (int k = 1; k <= kFaMaxRing; ++k) {
      if (fa_layout(D, k, v).total > budget) continue;
      // the deeper ring goes to V: a V entry is held from its load until the second MMA2 of the tile
      const int score = std::min(k, v) * 100 + k + 2 * v;
      if (best_k == 0 || score > std::min(best_k, best_v) * 100 + best_k + 2 * best_v) {
        best_k = k;
        best_v = v;
      }
    }
  if (best_k == 0) return false;
  *nk = best_k;
  *nv = best_v;
  *num_ctas = num_sms;
  *smem_bytes = fa_layout(D, best_k, best_v).total + 1024;
  return true;
}

cudaError_t launch_fa_fwd(int D, int num_ctas, size_t smem, const CUtensorMap& mQ, const CUtensorMap& mK,
                          const CUtensorMap& mV, const CUtensorMap& mKs, const CUtensorMap& mVs,
                          const FaFwdParams& p, cudaStream_t stream) {
  if (D == 64) return fa_launch_t<64>(num_ctas, smem, mQ, mK, mV, mKs, mVs, p, stream);
  if (D == 128) return fa_launch_t<128>(num_ctas, smem, mQ, mK, mV, mKs, mVs, p, stream);
  return cudaErrorInvalidValue;
}

cudaError_t launch_fa_schedule(const FaFwdParams& p, int num_ctas, cudaStream_t stream) {
  fa_schedule_kernel<<<1, 1024, 0, stream>>>(p, num_ctas / ((p.group + 1) / 2), p.group);
  return cudaGetLastError();
}

cudaError_t launch_fa_combine(const FaFwdParams& p, int D, int max_streams, float* out, float* lse, float* mass,
                              cudaStream_t stream) {
  if (max_streams <= 0) return cudaSuccess;
  fa_combine_kernel<<<max_streams, 128, 0, stream>>>(p, D, p.group, out, lse, mass);
  return cudaGetLastError();
}

}  // namespace ska
