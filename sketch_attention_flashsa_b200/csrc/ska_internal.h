// Internal interfaces between the C-ABI host layer and the kernels of libska.so.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "../../include/sketch_attn.h"

namespace ska {

constexpr int kTileTokens = 128;       // history tokens per pipeline tile
constexpr int kMaxProtosPerCta = 256;  // prototypes one CTA holds in TMEM
constexpr uint64_t kDefaultBudgetNs = 4000000000ull;

// Workspace header (first 256 bytes of every workspace).
struct WsHeader {
  int32_t status;      // first device-side error (ska_status), 0 if none
  int32_t total_tiles; // written by the scheduling kernel
  int32_t tiles_per_cluster;
  int32_t pad[61];
};
static_assert(sizeof(WsHeader) == 256, "header is 256 bytes");

// Parameters of the prototype-wise (paper Eq. (8)) fused forward kernel.
struct ProtoFwdParams {
  const int32_t* cu_seqlens;   // [B+1]
  const int32_t* seqused;      // [B] or null
  const int32_t* tile_prefix;  // [B+1] exclusive prefix of per-user tile counts
  WsHeader* hdr;               // status + schedule
  float* partial;              // [(num_segments + num_clusters) * k * D] fp32
  float* lse;                  // [T, H] or null
  float* mass_partial;         // [(num_segments + num_clusters) * k] or null
  float* maxw;                 // [T, H] or null: each token's largest weight, 1 / L (Fig. 3 diagnostic)
  int B, H, k;
  int total_tokens;
  int q_per_user;
  int nk_slots;                // K ring: 16 KB slots
  int nv_entries;              // V ring: entries of D/64 x 16 KB
  float scale_log2;            // scale * log2(e)
  uint64_t budget_ns;
  uint32_t debug_flags;
};

struct ProtoFwdLaunch {
  int cluster;          // CTAs per cluster (prototype groups)
  int kc;               // prototypes per CTA
  int num_clusters;     // persistent clusters
  bool mass;            // the kernel also accumulates the per-prototype mass
  size_t smem_bytes;
};

// Host-side planning (no device access). With `mass` the CTAs hold at most 128 prototypes each,
// which leaves tensor memory for the mass accumulator.
bool proto_fwd_plan(int head_dim, int num_protos, int num_sms, bool mass, ProtoFwdLaunch* out, int* nk_slots,
                    int* nv_entries);

// Clusters of the planned configuration resident at once on the current device (0 if unknown).
int proto_fwd_max_clusters(int head_dim, const ProtoFwdLaunch& L);

cudaError_t launch_proto_fwd(int head_dim, const ProtoFwdLaunch& L, const CUtensorMap& mapQ,
                             const CUtensorMap& mapK, const CUtensorMap& mapV, const ProtoFwdParams& p,
                             cudaStream_t stream);

// Parameters of the row-softmax (FlashAttention-style) forward shared by token-wise SA and
// STCA. A "stream" is one 128-row query tile of one (user, head): prototypes (SA) or targets
// (STCA); its keys are the user's valid history (SA) or [suffix ; sketch] (STCA).
struct FaFwdParams {
  int mode;                    // 0 = SA token-wise, 1 = STCA
  const int32_t* cu_keys;      // SA: cu_seqlens; STCA: cu_hist
  const int32_t* seqused;      // SA only, nullable
  const int32_t* cu_q;         // STCA: cu_targets; SA: null
  const int32_t* kv_len;       // STCA: per-target suffix length, nullable
  const int32_t* tile_prefix;  // [B+1] key-tile columns (H per user) of users < b
  int group;                   // CTAs per group = query tiles walked together
  WsHeader* hdr;
  float* part_o;               // [(B*H + groups) * group * 128 * D] unnormalised O
  float* part_ml;              // [(B*H + groups) * group * 128 * 2] (max in log2 units, sum)
  int B, H;
  int k;                       // SA: prototypes
  int ks;                      // STCA: sketch rows per (user, head)
  int q_per_user;              // SA: q is [B,H,k,d]
  int nk_slots, nv_entries;
  float scale_log2;
  uint64_t budget_ns;
  uint32_t debug_flags;
};

bool fa_fwd_plan(int head_dim, int num_sms, int* num_ctas, size_t* smem_bytes, int* nk, int* nv);

cudaError_t launch_fa_fwd(int head_dim, int num_ctas, size_t smem_bytes, const CUtensorMap& mapQ,
                          const CUtensorMap& mapK, const CUtensorMap& mapV, const CUtensorMap& mapKs,
                          const CUtensorMap& mapVs, const FaFwdParams& p, cudaStream_t stream);

cudaError_t launch_fa_schedule(const FaFwdParams& p, int num_ctas, cudaStream_t stream);

// LSE merge of the partials into the outputs (max_streams = B * H * group blocks).
// SA: out = sketch [B,H,k,D], lse [B,H,k], mass [B,H,k] (nullable). STCA: out [total_targets, H, D],
// lse [total_targets, H], mass null.
cudaError_t launch_fa_combine(const FaFwdParams& p, int head_dim, int max_streams, float* out, float* lse,
                              float* mass, cudaStream_t stream);

// Parameters of the SA backward (both normalisations).
struct SaBwdParams {
  int norm;                    // SKA_NORM_PROTO or SKA_NORM_TOKEN
  const int32_t* cu_seqlens;
  const int32_t* seqused;
  const int32_t* tile_prefix;  // [B+1] (from launch_schedule)
  WsHeader* hdr;
  const float* lse;            // PROTO [T,H] (natural log); TOKEN [B,H,k]
  const float* sketch;         // TOKEN: forward output [B,H,k,d] (for D_j = dO_j . O_j)
  const __nv_bfloat16* dsketch;// [B,H,k,d] (TOKEN: D_j)
  float* dk;                   // [T,H,d]
  float* dv;                   // [T,H,d]
  float* dq_partial;           // [(B*H + ctas) * k * d], k = this launch's prototypes
  int B, H, k, total_tokens, q_per_user;
  float scale;
  uint64_t budget_ns;
};

// One launch over a chunk of a larger prototype set (its own kernel parameter: kept apart from
// SaBwdParams, whose size the register allocation of the fused kernel turned out sensitive to).
struct SaBwdChunk {
  float* delta;    // PROTO: [T,H], delta_i summed over the chunks
  int kt, j0;      // all prototypes, and the first one of this launch (one launch: k, 0)
  int pass;        // 0: every gradient; 1: PROTO delta_i only, this chunk's part added into
                   // delta; 2: every gradient with delta_i read from delta
  int accumulate;  // dK, dV added to the previous chunk's
};

bool sa_bwd_supported(int head_dim, int num_protos);
// Prototypes per launch: num_protos itself when one CTA holds them all, else the chunk size
// (128 for head_dim 128, 256 for 64) dividing num_protos; 0 if unsupported.
int sa_bwd_chunk(int head_dim, int num_protos);
size_t sa_bwd_smem_bytes(int head_dim, int num_protos);
cudaError_t launch_sa_bwd(int head_dim, int num_ctas, const CUtensorMap& mapQ, const CUtensorMap& mapDO,
                          const CUtensorMap& mapK, const CUtensorMap& mapV, const SaBwdParams& p,
                          const SaBwdChunk& ck, cudaStream_t stream);
// dq = scale * sum of the partial slots of every segment with head h (shared prototypes) or of
// segment (b, h) (per-user queries), in a fixed order; also zeroes dK/dV rows of padding tokens.
cudaError_t launch_sa_bwd_finish(const SaBwdParams& p, const SaBwdChunk& ck, int head_dim, float* dq,
                                 cudaStream_t stream);

// Parameters of the stacked refinement of the sketch (sa_refine.cu): rows (b, h, j) of
// [B, H, k, D] fp32 tensors; per-head LayerNorm vectors [H, D] (nullable: gamma 1, beta 0).
struct RefineParams {
  const float* x_tilde;
  const float* x_hat;
  const float* gamma1;
  const float* beta1;
  const float* gamma2;
  const float* beta2;
  float* x_bar;          // nullable: Eq. (13)'s output
  float* x_next;         // null in projection mode
  uint8_t* x_next_bf16;  // nullable: bf16 copy of x_next
  uint8_t* q_next;       // nullable: bf16 [B, H, k, D] = x_next W_Q (projection mode: x_tilde W_Q)
  int* status;           // the workspace status word
  int B, H, k;
  int x_tilde_shared;    // 1: x_tilde is [H, k, D], the same rows for every user
  int mode;              // 0: refinement (+ optional projection); 1: projection of x_tilde only
  float eps;
  uint64_t budget_ns;
  uint32_t debug_flags;  // bit 1 (value 2): never signal MMA1's completion (test hook)
};

bool sa_refine_supported(int head_dim, int ffn_dim);
// The fused refinement kernel on num_ctas persistent CTAs. mapWq is read only when p.q_next is set.
cudaError_t launch_sa_refine(int head_dim, int ffn_dim, int num_ctas, const CUtensorMap& mapW1,
                             const CUtensorMap& mapWg, const CUtensorMap& mapW2, const CUtensorMap& mapWq,
                             const RefineParams& p, cudaStream_t stream);
// Turns every output of the call to NaN when the status word holds an error (launched after it).
cudaError_t launch_refine_poison(int head_dim, const RefineParams& p, cudaStream_t stream);

// Parameters of the STCA backward (stca_bwd.cu).
struct StcaBwdParams {
  const int32_t* cu_q;     // cu_targets [B+1]
  const int32_t* cu_k;     // cu_hist [B+1]
  const int32_t* kv_len;   // [total_targets] or null
  const float* lse;        // [total_targets, H], natural log, from the forward
  float* delta;            // [total_targets, H] workspace: <dO, out>
  int32_t* kprefix;        // [B+1] workspace: H x key tiles of the users before b
  int32_t* qprefix;        // [B+1] workspace: H x target tiles of the users before b
  WsHeader* hdr;           // status; total_tiles = key items, tiles_per_cluster = target items
  float* dq;               // [total_targets, H, D]
  float* dk_hist;          // [total_hist, H, D]
  float* dv_hist;
  float* dk_sk;            // [B, H, ks, D]
  float* dv_sk;
  int B, H, ks;
  float scale;
  uint64_t budget_ns;
};

bool stca_bwd_supported(int head_dim);
// The schedule (item prefixes, status cleared) and delta = <dO, out> per (target, head).
cudaError_t launch_stca_bwd_prep(const StcaBwdParams& p, const void* dout, const float* out, int64_t rows,
                                 int head_dim, cudaStream_t stream);
// The key-major (dK, dV) then the query-major (dq) kernel. maps: Q, dO, K suffix, V suffix, K sketch,
// V sketch.
cudaError_t launch_stca_bwd(int head_dim, int ctas_kv, int ctas_q, const CUtensorMap* maps, const StcaBwdParams& p,
                            cudaStream_t stream);
// NaN into every gradient when the status word holds an error.
cudaError_t launch_stca_bwd_poison(const StcaBwdParams& p, int64_t n_dq, int64_t n_hist, int64_t n_sketch,
                                   cudaStream_t stream);

// Sketch cache (sketch_cache.cu).
bool cache_desc_ok(const ska_cache_desc* d);
size_t cache_bytes(const ska_cache_desc& d);
cudaError_t launch_cache_init(const ska_cache_desc& d, void* cache, cudaStream_t stream);
cudaError_t launch_cache_put(const ska_cache_desc& d, void* cache, const ska_cache_key* keys, const float* rows, int n,
                             int64_t now, int32_t* slots, cudaStream_t stream);
cudaError_t launch_cache_get(const ska_cache_desc& d, const void* cache, const ska_cache_key* keys, int n, int64_t now,
                             float* out, int32_t* hits, cudaStream_t stream);

// Small kernels (ska_small.cu).
cudaError_t launch_schedule(const int32_t* cu_seqlens, const int32_t* seqused, int B, int H,
                            int num_clusters, int32_t* tile_prefix, WsHeader* hdr, cudaStream_t stream);
// Also marks the call SKA_ERR_RANGE in hdr->status when a summed sketch value is not finite (an
// fp16 overflow of a scaled value row), and writes NaN when hdr->status reports an error.
// With `renormalize` every sketch row is divided by its prototype's mass (zero rows for zero mass).
cudaError_t launch_proto_combine(const int32_t* tile_prefix, WsHeader* hdr, const float* partial,
                                 const float* mass_partial, int B, int H, int k, int D, float* sketch,
                                 float* mass, bool renormalize, cudaStream_t stream);
// -inf lse and -1 maximum weight (either may be null) on the padding rows of every user.
cudaError_t launch_fill_padding_lse(const int32_t* cu_seqlens, const int32_t* seqused, int B, int H,
                                    int64_t T, float* lse, float* maxw, cudaStream_t stream);
// counts[b] (zeroed first) = number of values in [b / bins, (b + 1) / bins), 1.0 in the last bin;
// negative and NaN values are skipped.
cudaError_t launch_weight_histogram(const float* values, int64_t n, int bins, int32_t* counts, cudaStream_t stream);
cudaError_t launch_cast_f32_bf16(const float* src, void* dst, int64_t n, cudaStream_t stream);

}  // namespace ska
