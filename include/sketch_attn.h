/*
 * sketch_attn.h — C ABI of libska.so: Sketch Attention (SA) and STCA on NVIDIA B200 (sm_100a).
 *
 * The operations are those of "SequenceO1: End-to-End Ultra-Long (100K) Sequence Modeling in
 * Recommendation with Low-Rank Caching" (arXiv 2609.08443):
 *
 *   SA (§3.1, Eq. (7)-(9)): for a user with history keys K = X W_K (n x d) and values V (the
 *   history X itself in the paper) and prototypes Q = P W_Q (k x d),
 *       S = scale * Q K^T                         (k x n; the paper's scale is 1/sqrt(d))
 *       A = softmax_proto(S), sum_j A[j,i] = 1    (prototype-wise: over j for every token i)
 *       sketch = A V                              (k x d; fixed size, target-agnostic)
 *   FlashSA (§4.4) computes this in one streaming pass: block-wise affinities, softmax
 *   statistics (max and log-sum-exp) and aggregation, without storing the k x n scores.
 *
 *   SKA_NORM_TOKEN selects the token-wise ("vanilla attention") normalisation that §5.1 / Table 1
 *   compares against: A = softmax over the valid tokens i for every prototype j.
 *
 *   STCA (§2.3; used on the recent suffix and on the sketch in §3.4, batched per user by MRLB in
 *   §4.2): out_t = softmax(scale * q_t K^T) V over the keys [suffix rows of the target's user ;
 *   that user's sketch rows], one softmax per (target, head).
 *
 *   Stacked refinement (§3.3, Eq. (13)-(14)): after a layer's SA aggregation X^ the sketch is
 *   updated as LN(X~ + X^), then LN(. + FFN(.)) with a SwiGLU FFN (sa_refine).
 *
 * Heads: H heads are H independent problems on d-wide slices (the paper's SA is single-head).
 *
 * Conventions shared by every entry point
 *   Memory     All tensor arguments are DEVICE pointers owned by the caller, row-major and
 *              contiguous, 16-byte aligned. Integer index arrays are int32 on the device. The
 *              library never reads device memory from the host; sizes (total_*, max_*) come in
 *              the descriptor. The library allocates nothing: scratch memory is the caller's
 *              workspace `ws` of at least *_workspace_size() bytes (256-byte aligned).
 *   Execution  Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *              stream) and returns before the work finishes. Calls are reentrant; two calls must
 *              not share a workspace while both are in flight.
 *   Errors     Invalid arguments are reported before anything is launched (SKA_ERR_INVALID_VALUE,
 *              SKA_ERR_UNSUPPORTED, SKA_ERR_WORKSPACE_TOO_SMALL); a failed launch returns
 *              SKA_ERR_CUDA. A kernel that waits longer than its time budget on a pipeline
 *              barrier stops, records SKA_ERR_DEVICE_TIMEOUT in the workspace status word and
 *              exits; ska_read_device_status() reports it. Whenever a call's status word holds
 *              an error, that call's outputs are NaN, never plausible-looking values.
 *   Outputs    Outputs are fully overwritten (zeros for empty users). No output may alias an
 *              input. k and v may alias each other (the paper's V = X).
 *   Padding    Tokens of user b at positions >= seqused[b] take no part in the result, but their
 *              rows must hold finite numbers (a zero weight times a non-finite value is NaN).
 *   Precision  Scores S = scale Q K^T are exact products of the bf16 inputs summed in fp32; the
 *              softmax runs in fp32. SKA_NORM_PROTO aggregates in fp16 with fp32 accumulation:
 *              each value row v_i enters as fp16(w_i v_i), w_i the largest weight of token i
 *              among the prototypes of one CTA, times fp16 weights A / w_i in (0, 1]; this needs
 *              |w_i v_i| < 65520, else the product is infinite, the call records
 *              SKA_ERR_RANGE in the device status word and its outputs are NaN. SKA_NORM_TOKEN
 *              and STCA aggregate bf16 weights with the bf16 values in fp32.
 *   Determinism  Results are bitwise reproducible run to run (fixed-order reductions).
 */
#ifndef SKETCH_ATTN_H_
#define SKETCH_ATTN_H_

#include <stddef.h>
#include <stdint.h>

/* The library is built with hidden visibility; only the calls below are exported. */
#if defined(__GNUC__)
#define SKA_API __attribute__((visibility("default")))
#else
#define SKA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SKA_OK = 0,
  SKA_ERR_INVALID_VALUE = 1,       /* bad pointer, size, stride or alignment */
  SKA_ERR_UNSUPPORTED = 2,         /* valid but not implemented (e.g. head_dim not 64/128) */
  SKA_ERR_WORKSPACE_TOO_SMALL = 3, /* ws_bytes < *_workspace_size(desc) */
  SKA_ERR_CUDA = 4,                /* a CUDA runtime call or launch failed */
  SKA_ERR_DEVICE_TIMEOUT = 5,      /* a kernel gave up waiting on a pipeline barrier */
  SKA_ERR_RANGE = 6                /* a value is outside the range the kernel represents */
} ska_status;

typedef enum { SKA_BF16 = 0, SKA_F32 = 1 } ska_dtype;

typedef enum {
  SKA_NORM_PROTO = 0, /* the paper's Eq. (8): softmax over prototypes for every token */
  SKA_NORM_TOKEN = 1  /* §5.1 comparator: softmax over tokens for every prototype */
} ska_norm;

/* One batched SA problem: num_users ragged users, each with its own history.
 *   num_heads    H >= 1
 *   head_dim     d, 64 or 128
 *   num_protos   k >= 1. SKA_NORM_TOKEN: any k. SKA_NORM_PROTO: k / ceil(k / 256) in
 *                {16, 32, 64, 96, 128, 192, 256}, e.g. 16, 32, 64, 96, 128, 192, 256, 384, 512,
 *                576, 768, 1024; also 1536 and 2048 with head_dim 64 (with d = 128 the cluster
 *                exchange of k/256 CTAs does not fit shared memory); other k give
 *                SKA_ERR_UNSUPPORTED
 *   total_tokens rows of k and v (= cu_seqlens[num_users]); < 2^31
 *   max_seqlen   an upper bound on any user's length (informational; may be 0)
 *   scale        multiplies Q K^T; must be > 0 and finite (1/sqrt(d) in Eq. (7))
 *   norm         ska_norm
 *   in_dtype     ska_dtype of q, k, v (SKA_F32 inputs are rounded to bf16 in the workspace)
 *   q_per_user   0: q is [H, k, d], the prototypes shared by every user (layer 0, Eq. (6));
 *                1: q is [B, H, k, d], per-user queries (a refinement layer, §3.3)          */
typedef struct {
  int32_t num_users;
  int32_t num_heads;
  int32_t head_dim;
  int32_t num_protos;
  int64_t total_tokens;
  int32_t max_seqlen;
  float scale;
  int32_t norm;
  int32_t in_dtype;
  int32_t q_per_user;
  int32_t reserved;
} ska_sa_desc;

/* Bytes of workspace sa_forward needs for this descriptor (0 if the descriptor is invalid). */
SKA_API size_t sa_forward_workspace_size(const ska_sa_desc* desc);

/* SA forward (FlashSA), §3.1 Eq. (7)-(9) and §4.4.
 *   q           [H,k,d] or [B,H,k,d] (q_per_user), in_dtype
 *   k, v        [total_tokens, H, d], in_dtype; user b owns rows [cu_seqlens[b], cu_seqlens[b+1])
 *   cu_seqlens  int32 [B+1], non-decreasing, cu_seqlens[0] = 0
 *   seqused     int32 [B] or NULL: only the first min(seqused[b], len_b) rows of user b count
 *   sketch      out, fp32 [B, H, k, d]
 *   lse         out, fp32, may be NULL. PROTO: [total_tokens, H], the per-token log-sum-exp over
 *               the k prototypes (-inf on padding rows). TOKEN: [B, H, k], the per-prototype
 *               log-sum-exp over the valid tokens (-inf for an empty user). The backward pass
 *               needs it.
 *   mass        out, fp32 [B, H, k] or NULL: sum_i A[j,i] over the valid tokens, the mass each
 *               prototype received (PROTO: sum_j mass = the user's valid length; TOKEN: 1, or 0
 *               for an empty user). In PROTO mode a CTA then holds at most 128 prototypes,
 *               which limits k to 1024 and makes the call slower; without it (NULL) the call
 *               runs at full speed.                                                          */
SKA_API ska_status sa_forward(const ska_sa_desc* desc, const void* q, const void* k, const void* v,
                      const int32_t* cu_seqlens, const int32_t* seqused, float* sketch, float* lse,
                      float* mass, void* ws, size_t ws_bytes, void* stream);

/* SA forward with the allocation diagnostics (prototype-wise normalisation only; SKA_NORM_TOKEN
 * returns SKA_ERR_UNSUPPORTED). Arguments as in sa_forward (same workspace size), plus:
 *   token_max_weight  out, fp32 [total_tokens, H] or NULL: max_j A[j, i] for every token i, the
 *                     "maximum normalized weight" whose distribution §5.1 / Fig. 3 reports; it lies
 *                     in [1/k, 1]; -1 on padding rows
 *   renormalize       nonzero: the sketch rows become sum_i A[j,i] v_i / sum_i A[j,i], the
 *                     mass-weighted mean of the values (the Slot-Attention reading of the
 *                     normalisation that §2.4 compares SA with); zero rows for zero mass. mass must
 *                     then be given (it holds the divisors).                                      */
SKA_API ska_status sa_forward_diag(const ska_sa_desc* desc, const void* q, const void* k, const void* v,
                                   const int32_t* cu_seqlens, const int32_t* seqused, float* sketch, float* lse,
                                   float* mass, float* token_max_weight, int32_t renormalize, void* ws,
                                   size_t ws_bytes, void* stream);

/* Histogram of n fp32 values in [0, 1] (e.g. token_max_weight): counts[b], int32, zeroed by the call,
 * is the number of values in [b / bins, (b + 1) / bins), 1.0 counted in the last bin; negative
 * (padding) and NaN values are skipped. 1 <= bins <= 4096. Counts are exact (integer sums).     */
SKA_API ska_status sa_weight_histogram(const float* values, int64_t n, int32_t bins, int32_t* counts, void* stream);

/* Bytes of workspace sa_backward needs (0 if the descriptor is invalid). */
SKA_API size_t sa_backward_workspace_size(const ska_sa_desc* desc);

/* SA backward: gradients of <dsketch, sketch> through Eq. (7)-(9) (SA is trained end to end,
 * App. A.4). Inputs as in sa_forward (bf16 only), plus:
 *   sketch   fp32 [B, H, k, d], the forward output; read in TOKEN mode (D_j = dO_j . O_j), may
 *            be NULL in PROTO mode
 *   lse      fp32, the forward's lse (PROTO [total_tokens, H]; TOKEN [B, H, k])
 *   dsketch  bf16 [B, H, k, d]
 *   dq       out, fp32, q's shape: [H,k,d] summed over all users when the prototypes are shared,
 *            else [B,H,k,d]
 *   dk, dv   out, fp32 [total_tokens, H, d]; zero rows on padding tokens
 * Supported (SKA_ERR_UNSUPPORTED otherwise): num_protos in {16, 32, 64, 128, 256} for head_dim
 * 64 and {16, 32, 64, 128} for head_dim 128 in one fused launch; larger sets up to 4096 that are
 * multiples of 256 (head_dim 64) or 128 (head_dim 128) in one launch per chunk of that many
 * prototypes, dK and dV summed over the chunks in chunk order. In PROTO mode those first run
 * one pass per chunk for delta_i = sum_j A_ij dA_ij, kept in the workspace: 1.4x the FLOPs of
 * one fused pass, and the keys and values are read 2 k / chunk times (TOKEN: k / chunk). dQ is
 * formed from a two-term bf16 split of dS (16 significant bits), and over chunks so are dK (from
 * dS) and dV (from A); dQ is reduced over users in a fixed order. Results are bitwise
 * reproducible run to run.                                                                     */
SKA_API ska_status sa_backward(const ska_sa_desc* desc, const void* q, const void* k, const void* v,
                       const int32_t* cu_seqlens, const int32_t* seqused, const float* sketch,
                       const float* lse, const void* dsketch, float* dq, float* dk, float* dv, void* ws,
                       size_t ws_bytes, void* stream);

/* One batched STCA problem (§2.3, §3.4, MRLB §4.2): num_users users, each with a block of
 * target queries that share the user's keys.
 *   head_dim 64 or 128; num_sketch = k_s sketch rows per user (0 allowed);
 *   total_targets = cu_targets[B]; total_hist = cu_hist[B]; scale > 0 (1/sqrt(d_h) in §2.3);
 *   max_targets: an upper bound on any user's target count (0: total_targets is used, which is
 *   always a bound but leaves CTAs idle). A kernel that finds a user with more targets records
 *   SKA_ERR_INVALID_VALUE in the device status word and computes nothing. max_hist: unused.  */
typedef struct {
  int32_t num_users;
  int32_t num_heads;
  int32_t head_dim;
  int32_t num_sketch;
  int64_t total_targets;
  int64_t total_hist;
  int32_t max_targets;
  int32_t max_hist;
  float scale;
  int32_t reserved;
} ska_stca_desc;

SKA_API size_t stca_forward_workspace_size(const ska_stca_desc* desc);

/* STCA forward. All bf16 except the fp32 outputs.
 *   q              [total_targets, H, d]; targets of user b are rows [cu_targets[b], cu_targets[b+1])
 *   k_hist, v_hist [total_hist, H, d]; the recent suffix of user b is rows [cu_hist[b], cu_hist[b+1])
 *   target_kv_len  int32 [total_targets] or NULL: target t sees only the first target_kv_len[t]
 *                  suffix rows of its user (request-aware masking, §4.2)
 *   k_sk, v_sk     [B, H, num_sketch, d] (NULL when num_sketch == 0)
 *   out            fp32 [total_targets, H, d];  lse  fp32 [total_targets, H] or NULL          */
SKA_API ska_status stca_forward(const ska_stca_desc* desc, const void* q, const int32_t* cu_targets,
                        const void* k_hist, const void* v_hist, const int32_t* cu_hist,
                        const int32_t* target_kv_len, const void* k_sk, const void* v_sk, float* out,
                        float* lse, void* ws, size_t ws_bytes, void* stream);

/* Bytes of workspace stca_backward needs (0 if the descriptor is invalid). */
SKA_API size_t stca_backward_workspace_size(const ska_stca_desc* desc);

/* STCA backward: gradients of <dout, out> through stca_forward (STCA is trained end to end with
 * the ranker, §2.3; through its sketch branch the gradients reach the SA sketch, §3.4). Inputs as
 * in stca_forward, plus:
 *   out      fp32 [total_targets, H, d], the forward output (delta_t = <dout_t, out_t>)
 *   lse      fp32 [total_targets, H], the forward's lse
 *   dout     bf16 [total_targets, H, d]
 *   dq       out, fp32 [total_targets, H, d]
 *   dk_hist, dv_hist   out, fp32 [total_hist, H, d]: summed over the targets of the row's user
 *                      that see it (target_kv_len); zero for rows no target sees
 *   dk_sk, dv_sk       out, fp32 [B, H, num_sketch, d] (NULL when num_sketch == 0)
 * head_dim 64 or 128. max_targets and max_hist are not used. dq takes dS as a two-term bf16 split
 * (16 significant bits); dK and dV take P and dS in bf16, with fp32 accumulation.             */
SKA_API ska_status stca_backward(const ska_stca_desc* desc, const void* q, const int32_t* cu_targets,
                                 const void* k_hist, const void* v_hist, const int32_t* cu_hist,
                                 const int32_t* target_kv_len, const void* k_sk, const void* v_sk,
                                 const float* out, const float* lse, const void* dout, float* dq,
                                 float* dk_hist, float* dv_hist, float* dk_sk, float* dv_sk, void* ws,
                                 size_t ws_bytes, void* stream);

/* Stacked refinement of the sketch (§3.3, Eq. (13)-(14)): one layer's update of the per-user
 * sketch after its SA aggregation,
 *   x_bar  = LN1(x_tilde + x_hat)                               Eq. (13)
 *   x_next = LN2(x_bar + FFN(x_bar)),  FFN(U) = (swish(U W_1) * (U W_g)) W_2     Eq. (14)
 * with the SwiGLU FFN of App. G.1 (swish(u) = u sigmoid(u)) at the intermediate width ffn_dim =
 * 2 head_dim of App. G.3. Each LayerNorm normalises one row over its head_dim features with the
 * biased variance and eps, then applies gamma and beta. Head h uses its own weights and LayerNorm
 * vectors, as the SA call treats heads as independent problems.
 *   num_users B >= 0, num_heads H >= 1, num_protos k >= 1 (the sketch rows of one user and head;
 *   any k), head_dim 64 or 128, ffn_dim = 2 head_dim (other pairs: SKA_ERR_UNSUPPORTED), eps > 0
 *   and finite. B * H * k * head_dim < 2^31.
 *   x_tilde_shared  0: x_tilde is [B, H, k, d]; 1: x_tilde is [H, k, d], one set of rows for every
 *                   user (layer 0, whose X~ is the prototypes P^(0)).                           */
typedef struct {
  int32_t num_users;
  int32_t num_heads;
  int32_t num_protos;
  int32_t head_dim;
  int32_t ffn_dim;
  float eps;
  int32_t x_tilde_shared;
  int32_t reserved;
} ska_refine_desc;

/* Bytes of workspace sa_refine needs: 256, the status word (0 if the descriptor is invalid). */
SKA_API size_t sa_refine_workspace_size(const ska_refine_desc* desc);

/* Refinement layer. Device pointers; shapes for B users, H heads, k rows, d = head_dim, F = ffn_dim:
 *   x_tilde          fp32 [B, H, k, d] (or [H, k, d] with x_tilde_shared): the layer's input sketch
 *   x_hat            fp32 [B, H, k, d]: its SA output (sa_forward's sketch)
 *   w1, wg           bf16 [H, d, F];  w2  bf16 [H, F, d]
 *   gamma1, beta1, gamma2, beta2   fp32 [H, d] or NULL (NULL: gamma = 1, beta = 0)
 *   w_q_next         bf16 [H, d, d] or NULL: the next layer's query weights W_Q^(l+1)
 *   x_next           out, fp32 [B, H, k, d]
 *   x_bar            out, fp32 [B, H, k, d], or NULL when not wanted
 *   x_next_bf16      out, bf16 [B, H, k, d], or NULL: a bf16 copy of x_next
 *   q_next           out, bf16 [B, H, k, d], or NULL: x_next W_Q^(l+1) for each head, the per-user
 *                    queries of the next layer (Eq. (10); pass them to sa_forward with
 *                    q_per_user = 1 and scale 1/sqrt(d)). w_q_next and q_next come together.
 * The LayerNorms, the residual sums and swish run in fp32. The products with the weights take
 * their activations as a two-term bf16 split (16 significant bits) against the bf16 weights,
 * with fp32 accumulation; q_next is rounded to bf16 at the end. B = 0 returns SKA_OK without
 * launching anything.                                                                           */
SKA_API ska_status sa_refine(const ska_refine_desc* desc, const float* x_tilde, const float* x_hat,
                             const void* w1, const void* wg, const void* w2, const float* gamma1,
                             const float* beta1, const float* gamma2, const float* beta2,
                             const void* w_q_next, float* x_next, float* x_bar, void* x_next_bf16,
                             void* q_next, void* ws, size_t ws_bytes, void* stream);

/* Query projection of sketch rows, q = x W_Q per head (Eq. (7)'s P^(0) W_Q for layer 0, Eq. (10)'s
 * X~^(l) W_Q^(l) otherwise); the same kernel and precision as sa_refine's q_next.
 *   x      fp32 [num_users, num_heads, num_rows, head_dim]   (num_users = 1 for the prototypes)
 *   w_q    bf16 [num_heads, head_dim, head_dim]
 *   q_out  out, bf16, x's shape
 *   ws     at least 256 bytes (the device status word; ska_read_device_status reads it)
 * head_dim 64 or 128 (else SKA_ERR_UNSUPPORTED); num_heads, num_rows >= 1; num_users = 0 is a
 * no-op.                                                                                        */
SKA_API ska_status sa_project_queries(int32_t num_users, int32_t num_heads, int32_t num_rows, int32_t head_dim,
                                      const float* x, const void* w_q, void* q_out, void* ws,
                                      size_t ws_bytes, void* stream);

/* Sketch cache (§4.1): the user-only sketch X~_u (any fixed number of floats per user, e.g.
 * H x k x d) cached in device memory, keyed by user id, model version, history timestamp and sketch
 * configuration, with TTL invalidation and capacity eviction, one get/put interface for training
 * and serving.
 * Layout: num_sets sets (a power of two, <= 2^24) of `ways` ways (1..32); a key's set is SplitMix64
 * folded over the four key fields (user id, version, configuration, timestamp, in that order, each
 * mixed in by xor), masked to num_sets - 1. Times are the caller's integer clock (e.g. seconds);
 * an entry stored at time t is live while now - t <= ttl.
 *   get: a key hits when a way of its set holds it live; its row is copied out (a miss: zeros).
 *   put: keys are applied in batch order: a way holding the same key is overwritten, else the
 *        first empty or expired way is used, else the oldest (ties: the lowest way).
 * The cache memory is the caller's (sa_cache_bytes, 256-byte aligned); calls on one cache must be
 * ordered on one stream. row_floats is a multiple of 4; rows are 16-byte aligned.                 */
typedef struct {
  uint64_t user_id;
  uint32_t model_version;
  uint32_t sketch_config;
  int64_t history_timestamp;
} ska_cache_key;

typedef struct {
  int32_t num_sets;
  int32_t ways;
  int32_t row_floats;
  int32_t reserved;
  int64_t ttl;
} ska_cache_desc;

/* Bytes of device memory a cache needs (0 if the descriptor is invalid). */
SKA_API size_t sa_cache_bytes(const ska_cache_desc* desc);
/* Marks every way empty. */
SKA_API ska_status sa_cache_init(const ska_cache_desc* desc, void* cache, size_t cache_bytes, void* stream);
/* keys: device array of n keys; rows: fp32 [n, row_floats]; slots: out, int32 [n], the slot
 * (set * ways + way) each key was written to. */
SKA_API ska_status sa_cache_put(const ska_cache_desc* desc, void* cache, size_t cache_bytes, const ska_cache_key* keys,
                                const float* rows, int32_t n, int64_t now, int32_t* slots, void* stream);
/* out: fp32 [n, row_floats]; hits: out, int32 [n], 1 for a hit and 0 for a miss. */
SKA_API ska_status sa_cache_get(const ska_cache_desc* desc, const void* cache, size_t cache_bytes,
                                const ska_cache_key* keys, int32_t n, int64_t now, float* out, int32_t* hits,
                                void* stream);

/* Human-readable name of a status code (static string). */
SKA_API const char* ska_status_string(ska_status status);

/* Text of the last failure this host thread's calls recorded (the CUDA error behind an
 * SKA_ERR_CUDA return, or the step that failed); an empty string if none. Static, per thread. */
SKA_API const char* ska_last_error_string(void);

/* Reads the device status word of a workspace after synchronising `stream`; returns SKA_OK or
 * the first device-side error a kernel recorded there (e.g. SKA_ERR_DEVICE_TIMEOUT), and
 * clears it. Test and debug helper: it blocks the host. */
SKA_API ska_status ska_read_device_status(void* ws, void* stream);

/* Test hook (process-wide, not synchronised with concurrent calls): the time budget in ns of
 * every barrier wait in later launches (0 restores the default of 4 s), and debug flags
 * (1 = the load producer of later SA forward launches withholds its first arrival; 2 = later
 * sa_refine launches never signal that their first matrix products are done; either way the
 * kernels' bounded waits must run out and report SKA_ERR_DEVICE_TIMEOUT). */
SKA_API void ska_set_debug(uint64_t wait_budget_ns, uint32_t flags);

/* SA forward for callers that cannot allocate device memory (code running inside a memory
 * pool it does not own, plugins that only receive input and output pointers, service paths
 * that must not allocate after start-up). The paper has no counterpart: this is a deployment
 * variant of sa_forward. It runs the same kernels with its scratch memory in a file-scope
 * device array of sa_forward_noalloc_scratch_bytes() bytes (40 MiB) that every GPU loading this
 * library holds until the process exits; it calls no allocator.
 *   Arguments and outputs are those of sa_forward, without the workspace.
 *   Returns SKA_ERR_WORKSPACE_TOO_SMALL, before any launch, when the problem needs more scratch
 *   than the array holds (sa_forward_workspace_size(desc) > sa_forward_noalloc_scratch_bytes()).
 *   The first call on a device looks up the array's address (cudaGetSymbolAddress); make it
 *   before any stream capture. All calls on a device share the array: calls that overlap on
 *   the GPU (other streams, other host threads) race and must be serialised by the caller.   */
SKA_API ska_status sa_forward_noalloc(const ska_sa_desc* desc, const void* q, const void* k, const void* v,
                              const int32_t* cu_seqlens, const int32_t* seqused, float* sketch,
                              float* lse, float* mass, void* stream);

/* Size in bytes of the device array that sa_forward_noalloc uses as scratch. */
SKA_API size_t sa_forward_noalloc_scratch_bytes(void);

/* Device status of the sa_forward_noalloc calls on the current device: synchronises `stream`,
 * then returns SKA_OK or the first device-side error the last call recorded in the shared
 * array's status word (e.g. SKA_ERR_DEVICE_TIMEOUT, SKA_ERR_RANGE) and clears it. The next
 * sa_forward_noalloc call clears the word itself, so read it before that call. Blocks the host.
 * Returns SKA_ERR_CUDA when the array cannot be reached (no usable device).                  */
SKA_API ska_status sa_forward_noalloc_read_status(void* stream);

/* Bench hook (process-wide): while both handles are non-NULL, every later call records
 * `start_event` on its stream immediately before its fused main kernel and `stop_event`
 * immediately after it (cudaEvent_t handles created by the caller), so that the main kernel
 * can be timed on its own stream with CUDA events. Pass NULL, NULL to stop recording. */
SKA_API void ska_set_timing_events(void* start_event, void* stop_event);

#ifdef __cplusplus
}
#endif

#endif /* SKETCH_ATTN_H_ */
