// C-ABI host layer of libska.so: argument validation, workspace carving, TMA descriptor
// encoding and kernel launches. Everything here runs on the host and only enqueues work on
// the caller's stream; no device memory is read or allocated.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>

#include <cudaTypedefs.h>

#include "ska_internal.h"

using namespace ska;

namespace {

thread_local char g_last_error[256] = "";

void record_error(const char* what, cudaError_t e) {
  std::snprintf(g_last_error, sizeof(g_last_error), "%s: %s", what,
                e == cudaSuccess ? "failed" : cudaGetErrorString(e));
}

std::atomic<uint64_t> g_budget_ns{0};
std::atomic<uint32_t> g_debug_flags{0};
std::atomic<void*> g_ev_start{nullptr};
std::atomic<void*> g_ev_stop{nullptr};

struct TimedRegion {
  cudaStream_t s;
  cudaEvent_t stop;
  explicit TimedRegion(cudaStream_t st) : s(st), stop(nullptr) {
    cudaEvent_t a = static_cast<cudaEvent_t>(g_ev_start.load(std::memory_order_relaxed));
    cudaEvent_t b = static_cast<cudaEvent_t>(g_ev_stop.load(std::memory_order_relaxed));
    if (a && b) {
      cudaEventRecord(a, s);
      stop = b;
    }
  }
  ~TimedRegion() {
    if (stop) cudaEventRecord(stop, s);
  }
};

uint64_t wait_budget() {
  const uint64_t b = g_budget_ns.load(std::memory_order_relaxed);
  return b ? b : kDefaultBudgetNs;
}

int device_sm_count() {
  static int cache[64];
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  std::lock_guard<std::mutex> lock(mu);
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cache[dev] = n;
  }
  return cache[dev];
}

// True (and the reason recorded) when no CUDA device is usable from this thread.
bool no_device() {
  int dev = 0;
  if (cudaError_t e = cudaGetDevice(&dev); e != cudaSuccess) {
    cudaGetLastError();
    record_error("cudaGetDevice", e);
    return true;
  }
  if (device_sm_count() == 0) {
    record_error("cudaDeviceGetAttribute(multiProcessorCount)", cudaErrorInvalidDevice);
    return true;
  }
  return false;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D bf16 map over a row-major [rows, inner] tensor with 128-byte swizzle.
bool encode_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t row_stride_elems,
               uint32_t box_inner, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) {
    std::snprintf(g_last_error, sizeof(g_last_error), "cuTensorMapEncodeTiled: driver entry point not found");
    return false;
  }
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {row_stride_elems * 2};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t es[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    std::snprintf(g_last_error, sizeof(g_last_error), "cuTensorMapEncodeTiled: CUresult %d (inner %llu, rows %llu, box %u x %u)",
                  int(r), (unsigned long long)inner, (unsigned long long)rows, box_inner, box_rows);
  return r == CUDA_SUCCESS;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  if (!a || !b || na == 0 || nb == 0) return false;
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return a0 < b0 + nb && b0 < a0 + na;
}

// Validation shared by forward and backward descriptors.
ska_status check_sa_desc(const ska_sa_desc* d) {
  if (!d) return SKA_ERR_INVALID_VALUE;
  if (d->num_users < 0 || d->num_heads < 1 || d->total_tokens < 0 || d->total_tokens >= (int64_t(1) << 31))
    return SKA_ERR_INVALID_VALUE;
  if (!(d->scale > 0.f) || !std::isfinite(d->scale)) return SKA_ERR_INVALID_VALUE;
  if (d->norm != SKA_NORM_PROTO && d->norm != SKA_NORM_TOKEN) return SKA_ERR_INVALID_VALUE;
  if (d->in_dtype != SKA_BF16 && d->in_dtype != SKA_F32) return SKA_ERR_INVALID_VALUE;
  if (d->q_per_user != 0 && d->q_per_user != 1) return SKA_ERR_INVALID_VALUE;
  if (d->num_protos < 1) return SKA_ERR_INVALID_VALUE;
  if (d->head_dim != 64 && d->head_dim != 128) return SKA_ERR_UNSUPPORTED;
  if (int64_t(d->num_users) * d->num_heads >= (int64_t(1) << 30)) return SKA_ERR_INVALID_VALUE;
  // The concatenated tile stream (H * sum_b ceil(len_b / 128) <= H * (T / 128 + B)) is indexed
  // with 32-bit integers on the device.
  if (int64_t(d->num_heads) * (d->total_tokens / 128 + d->num_users + 1) >= (int64_t(1) << 31))
    return SKA_ERR_INVALID_VALUE;
  return SKA_OK;
}

struct FwdWs {
  size_t hdr, prefix, partial, mass_partial, qb, kb, vb, total;
};

bool fwd_ws_layout(const ska_sa_desc* d, const ProtoFwdLaunch& L, FwdWs* w) {
  const size_t B = d->num_users, H = d->num_heads, D = d->head_dim, k = d->num_protos;
  const size_t T = d->total_tokens;
  const size_t slots = B * H + L.num_clusters;
  size_t off = 0;
  w->hdr = off;
  off += sizeof(WsHeader);
  w->prefix = off;
  off = align256(off + (B + 1) * 4);
  w->partial = off;
  off = align256(off + slots * k * D * 4);
  w->mass_partial = off;
  off = align256(off + slots * k * 4);
  w->qb = w->kb = w->vb = 0;
  if (d->in_dtype == SKA_F32) {
    const size_t qn = (d->q_per_user ? B : 1) * H * k * D;
    w->qb = off;
    off = align256(off + qn * 2);
    w->kb = off;
    off = align256(off + T * H * D * 2);
    w->vb = off;
    off = align256(off + T * H * D * 2);
  }
  w->total = off;
  return true;
}

bool plan_forward(const ska_sa_desc* d, bool mass, ProtoFwdLaunch* L, int* nk, int* nv) {
  const int sms = device_sm_count();
  if (sms <= 0) return false;
  if (!proto_fwd_plan(d->head_dim, d->num_protos, sms, mass, L, nk, nv)) return false;
  // persistent clusters: no more than the device holds at once (a second wave would double the time)
  const int resident = proto_fwd_max_clusters(d->head_dim, *L);
  if (resident > 0 && resident < L->num_clusters) L->num_clusters = resident;
  return true;
}

// ---------------------------------------------------------------- row-softmax engine (token SA, STCA)
struct FaWs {
  size_t hdr, tile_prefix, part_o, part_ml, qb, kb, vb, total;
};

// Slots: one per (column stream (b, h) + group, query tile) pair along the column staircase.
void fa_ws_layout(int B, int H, int D, int G, int ngroups, size_t cast_q, size_t cast_kv, FaWs* w) {
  size_t off = 0;
  w->hdr = off;
  off += sizeof(WsHeader);
  w->tile_prefix = off;
  off = align256(off + size_t(B + 1) * 4);
  const size_t slots = (size_t(B) * H + size_t(ngroups)) * size_t(G);
  w->part_o = off;
  off = align256(off + slots * 128 * D * 4);
  w->part_ml = off;
  off = align256(off + slots * 128 * 2 * 4);
  w->qb = w->kb = w->vb = 0;
  if (cast_q || cast_kv) {
    w->qb = off;
    off = align256(off + cast_q * 2);
    w->kb = off;
    off = align256(off + cast_kv * 2);
    w->vb = off;
    off = align256(off + cast_kv * 2);
  }
  w->total = off;
}

// CTA count of the row-softmax engine for G query tiles walked together: groups of (G + 1) / 2
// CTAs, each CTA holding two query tiles.
bool fa_groups(int G, int sms, int* ctas, int* ngroups) {
  const int Gc = (G + 1) / 2;
  if (G < 1 || Gc > sms) return false;
  *ngroups = sms / Gc;
  *ctas = *ngroups * Gc;
  return true;
}

int sa_token_group(const ska_sa_desc* d) { return (d->num_protos + 127) / 128; }

size_t sa_token_ws_size(const ska_sa_desc* d, FaWs* w, int* ctas, size_t* smem, int* nk, int* nv) {
  const int sms = device_sm_count();
  int c0, ng;
  if (sms <= 0 || !fa_fwd_plan(d->head_dim, sms, &c0, smem, nk, nv)) return 0;
  const int G = sa_token_group(d);
  if (!fa_groups(G, sms, ctas, &ng)) return 0;
  const size_t qn = size_t(d->q_per_user ? d->num_users : 1) * d->num_heads * d->num_protos * d->head_dim;
  const size_t kvn = size_t(d->total_tokens) * d->num_heads * d->head_dim;
  fa_ws_layout(d->num_users, d->num_heads, d->head_dim, G, ng, d->in_dtype == SKA_F32 ? qn : 0,
               d->in_dtype == SKA_F32 ? kvn : 0, w);
  return w->total;
}

ska_status sa_forward_token(const ska_sa_desc* d, const void* q, const void* k, const void* v,
                            const int32_t* cu_seqlens, const int32_t* seqused, float* sketch, float* lse,
                            float* mass, void* ws, size_t ws_bytes, cudaStream_t s) {
  const int B = d->num_users, H = d->num_heads, D = d->head_dim, kp = d->num_protos;
  const int64_t T = d->total_tokens;
  FaWs w;
  int ctas, nk, nv;
  size_t smem;
  if (sa_token_ws_size(d, &w, &ctas, &smem, &nk, &nv) == 0) return SKA_ERR_UNSUPPORTED;
  if (ws_bytes < w.total) return SKA_ERR_WORKSPACE_TOO_SMALL;
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  const size_t qn = size_t(d->q_per_user ? B : 1) * H * kp * D;
  const size_t kvn = size_t(T) * H * D;
  const void* qb = q;
  const void* kb = k;
  const void* vb = v;
  if (d->in_dtype == SKA_F32) {
    if (launch_cast_f32_bf16(static_cast<const float*>(q), wsb + w.qb, int64_t(qn), s) != cudaSuccess ||
        launch_cast_f32_bf16(static_cast<const float*>(k), wsb + w.kb, int64_t(kvn), s) != cudaSuccess ||
        launch_cast_f32_bf16(static_cast<const float*>(v), wsb + w.vb, int64_t(kvn), s) != cudaSuccess)
      return SKA_ERR_CUDA;
    qb = wsb + w.qb;
    kb = wsb + w.kb;
    vb = wsb + w.vb;
  }
  FaFwdParams p{};
  p.mode = 0;
  p.cu_keys = cu_seqlens;
  p.seqused = seqused;
  p.cu_q = nullptr;
  p.kv_len = nullptr;
  p.tile_prefix = reinterpret_cast<int32_t*>(wsb + w.tile_prefix);
  p.group = sa_token_group(d);
  p.hdr = reinterpret_cast<WsHeader*>(wsb + w.hdr);
  p.part_o = reinterpret_cast<float*>(wsb + w.part_o);
  p.part_ml = reinterpret_cast<float*>(wsb + w.part_ml);
  p.B = B;
  p.H = H;
  p.k = kp;
  p.ks = 0;
  p.q_per_user = d->q_per_user;
  p.nk_slots = nk;
  p.nv_entries = nv;
  p.scale_log2 = d->scale * 1.4426950408889634f;
  p.budget_ns = wait_budget();
  p.debug_flags = g_debug_flags.load(std::memory_order_relaxed);
  if (cudaError_t e_ = launch_fa_schedule(p, ctas, s); e_ != cudaSuccess) { record_error("launch_fa_schedule", e_); return SKA_ERR_CUDA; }
  if (T > 0) {
    CUtensorMap mQ, mK, mV;
    const uint64_t qrows = uint64_t(d->q_per_user ? B : 1) * H * kp;
    if (!encode_2d(&mQ, qb, D, qrows, D, 64, 128)) return SKA_ERR_CUDA;
    if (!encode_2d(&mK, kb, uint64_t(H) * D, T, uint64_t(H) * D, 64, 128)) return SKA_ERR_CUDA;
    if (!encode_2d(&mV, vb, uint64_t(H) * D, T, uint64_t(H) * D, 64, 128)) return SKA_ERR_CUDA;
    cudaError_t e;
    {
      TimedRegion tr(s);
      e = launch_fa_fwd(D, ctas, smem, mQ, mK, mV, mK, mV, p, s);
    }
    if (e != cudaSuccess) {
      record_error("fused kernel launch", e);
      return SKA_ERR_CUDA;
    }
  }
  if (cudaError_t e_ = launch_fa_combine(p, D, B * H * p.group, sketch, lse, mass, s); e_ != cudaSuccess) { record_error("launch_fa_combine", e_); return SKA_ERR_CUDA; }
  return SKA_OK;
}

ska_status check_stca_desc(const ska_stca_desc* d) {
  if (!d) return SKA_ERR_INVALID_VALUE;
  if (d->num_users < 0 || d->num_heads < 1 || d->num_sketch < 0 || d->total_targets < 0 || d->total_hist < 0 ||
      d->total_targets >= (int64_t(1) << 31) || d->total_hist >= (int64_t(1) << 31))
    return SKA_ERR_INVALID_VALUE;
  if (!(d->scale > 0.f) || !std::isfinite(d->scale)) return SKA_ERR_INVALID_VALUE;
  if (d->head_dim != 64 && d->head_dim != 128) return SKA_ERR_UNSUPPORTED;
  if (int64_t(d->num_users) * d->num_heads * std::max(d->num_sketch, 1) >= (int64_t(1) << 31))
    return SKA_ERR_INVALID_VALUE;
  // key-tile columns: H * sum_b (ceil(hist_b / 128) + ceil(ks / 128)), 32-bit on the device
  if (int64_t(d->num_heads) * (d->total_hist / 128 + int64_t(d->num_users) * (d->num_sketch / 128 + 2) + 1) >=
      (int64_t(1) << 31))
    return SKA_ERR_INVALID_VALUE;
  return SKA_OK;
}

// Query tiles walked together: from max_targets when given (an upper bound on any user's target
// count), else from total_targets (always an upper bound, at the cost of idle CTAs).
int stca_group(const ska_stca_desc* d) {
  const int64_t mt = d->max_targets > 0 ? d->max_targets : d->total_targets;
  return int((mt + 127) / 128);
}

size_t stca_ws_size(const ska_stca_desc* d, FaWs* w, int* ctas, size_t* smem, int* nk, int* nv) {
  const int sms = device_sm_count();
  int c0, ng;
  if (sms <= 0 || !fa_fwd_plan(d->head_dim, sms, &c0, smem, nk, nv)) return 0;
  if (!fa_groups(stca_group(d), sms, ctas, &ng)) return 0;
  fa_ws_layout(d->num_users, d->num_heads, d->head_dim, stca_group(d), ng, 0, 0, w);
  return w->total;
}
}  // namespace

ska_status check_refine_desc(const ska_refine_desc* d) {
  if (!d) return SKA_ERR_INVALID_VALUE;
  if (d->num_users < 0 || d->num_heads < 1 || d->num_protos < 1) return SKA_ERR_INVALID_VALUE;
  if (!(d->eps > 0.f) || !std::isfinite(d->eps)) return SKA_ERR_INVALID_VALUE;
  if (!sa_refine_supported(d->head_dim, d->ffn_dim)) return SKA_ERR_UNSUPPORTED;
  if (int64_t(d->num_users) * d->num_heads * d->num_protos * d->head_dim >= (int64_t(1) << 31))
    return SKA_ERR_INVALID_VALUE;
  return SKA_OK;
}

extern "C" {

const char* ska_last_error_string(void) { return g_last_error; }

const char* ska_status_string(ska_status s) {
  switch (s) {
    case SKA_OK: return "SKA_OK";
    case SKA_ERR_INVALID_VALUE: return "SKA_ERR_INVALID_VALUE";
    case SKA_ERR_UNSUPPORTED: return "SKA_ERR_UNSUPPORTED";
    case SKA_ERR_WORKSPACE_TOO_SMALL: return "SKA_ERR_WORKSPACE_TOO_SMALL";
    case SKA_ERR_CUDA: return "SKA_ERR_CUDA";
    case SKA_ERR_DEVICE_TIMEOUT: return "SKA_ERR_DEVICE_TIMEOUT";
    case SKA_ERR_RANGE: return "SKA_ERR_RANGE";
  }
  return "SKA_ERR_UNKNOWN";
}

void ska_set_timing_events(void* start_event, void* stop_event) {
  g_ev_start.store(start_event, std::memory_order_relaxed);
  g_ev_stop.store(stop_event, std::memory_order_relaxed);
}

void ska_set_debug(uint64_t wait_budget_ns, uint32_t flags) {
  g_budget_ns.store(wait_budget_ns, std::memory_order_relaxed);
  g_debug_flags.store(flags, std::memory_order_relaxed);
}

ska_status ska_read_device_status(void* ws, void* stream) {
  if (!ws) return SKA_ERR_INVALID_VALUE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t v = 0;
  if (cudaMemcpyAsync(&v, ws, sizeof(v), cudaMemcpyDeviceToHost, st) != cudaSuccess) return SKA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return SKA_ERR_CUDA;
  if (v != 0) {
    const int32_t zero = 0;
    if (cudaMemcpyAsync(ws, &zero, sizeof(zero), cudaMemcpyHostToDevice, st) != cudaSuccess) return SKA_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return SKA_ERR_CUDA;
  }
  return static_cast<ska_status>(v);
}

size_t sa_forward_workspace_size(const ska_sa_desc* d) {
  if (check_sa_desc(d) != SKA_OK) return 0;
  if (d->norm == SKA_NORM_TOKEN) {
    FaWs w;
    int c, nk, nv;
    size_t sm;
    return sa_token_ws_size(d, &w, &c, &sm, &nk, &nv);
  }
  // Enough for the call with or without the mass output (their plans differ in cluster count,
  // hence in partial slots).
  ProtoFwdLaunch L;
  int nk, nv;
  if (!plan_forward(d, false, &L, &nk, &nv)) return 0;
  FwdWs w;
  fwd_ws_layout(d, L, &w);
  size_t total = w.total;
  if (plan_forward(d, true, &L, &nk, &nv)) {
    fwd_ws_layout(d, L, &w);
    total = std::max(total, w.total);
  }
  return total;
}

// sa_forward, plus (prototype-wise only) each token's largest weight and the mass-renormalised sketch.
static ska_status sa_forward_impl(const ska_sa_desc* d, const void* q, const void* k, const void* v,
                                  const int32_t* cu_seqlens, const int32_t* seqused, float* sketch, float* lse,
                                  float* mass, float* maxw, bool renormalize, void* ws, size_t ws_bytes, void* stream) {
  ska_status st = check_sa_desc(d);
  if (st != SKA_OK) return st;
  const int B = d->num_users, H = d->num_heads, D = d->head_dim, kp = d->num_protos;
  const int64_t T = d->total_tokens;
  if ((maxw || renormalize) && d->norm != SKA_NORM_PROTO) return SKA_ERR_UNSUPPORTED;
  if (B == 0) return SKA_OK;
  // pointers and alignment
  if (!q || !cu_seqlens || !sketch || !ws) return SKA_ERR_INVALID_VALUE;
  if (T > 0 && (!k || !v)) return SKA_ERR_INVALID_VALUE;
  if (renormalize && !mass) return SKA_ERR_INVALID_VALUE;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(sketch) || !aligned16(lse) ||
      !aligned16(mass) || !aligned16(maxw) || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0 ||
      (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) || (reinterpret_cast<uintptr_t>(seqused) & 3u))
    return SKA_ERR_INVALID_VALUE;
  // outputs against inputs and each other (host-only checks, before any device query)
  const size_t esz = d->in_dtype == SKA_F32 ? 4 : 2;
  const size_t qn = size_t(d->q_per_user ? B : 1) * H * kp * D;
  const size_t kvn = size_t(T) * H * D;
  const size_t sk_bytes = size_t(B) * H * kp * D * 4;
  const size_t lse_bytes = (d->norm == SKA_NORM_PROTO ? size_t(T) : size_t(B) * kp) * H * 4;
  const size_t mass_bytes = size_t(B) * H * kp * 4;
  if (overlaps(sketch, sk_bytes, q, qn * esz) || overlaps(sketch, sk_bytes, k, kvn * esz) ||
      overlaps(sketch, sk_bytes, v, kvn * esz) || overlaps(lse, lse_bytes, q, qn * esz) ||
      overlaps(lse, lse_bytes, k, kvn * esz) || overlaps(lse, lse_bytes, v, kvn * esz) ||
      overlaps(lse, lse_bytes, sketch, sk_bytes) || overlaps(mass, mass_bytes, q, qn * esz) ||
      overlaps(mass, mass_bytes, k, kvn * esz) || overlaps(mass, mass_bytes, v, kvn * esz) ||
      overlaps(mass, mass_bytes, sketch, sk_bytes) || overlaps(mass, mass_bytes, lse, lse_bytes))
    return SKA_ERR_INVALID_VALUE;
  const size_t mw_bytes = size_t(T) * H * 4;
  if (overlaps(maxw, mw_bytes, q, qn * esz) || overlaps(maxw, mw_bytes, k, kvn * esz) ||
      overlaps(maxw, mw_bytes, v, kvn * esz) || overlaps(maxw, mw_bytes, sketch, sk_bytes) ||
      overlaps(maxw, mw_bytes, lse, lse_bytes) || overlaps(maxw, mw_bytes, mass, mass_bytes))
    return SKA_ERR_INVALID_VALUE;
  if (no_device()) return SKA_ERR_CUDA;
  const size_t ws_need = sa_forward_workspace_size(d);
  if (ws_need == 0) return SKA_ERR_UNSUPPORTED;
  if (ws_bytes < ws_need) return SKA_ERR_WORKSPACE_TOO_SMALL;
  if (overlaps(ws, ws_need, sketch, sk_bytes) || overlaps(ws, ws_need, lse, lse_bytes) ||
      overlaps(ws, ws_need, q, qn * esz) || overlaps(ws, ws_need, k, kvn * esz) ||
      overlaps(ws, ws_need, v, kvn * esz) || overlaps(mass, mass_bytes, ws, ws_need) ||
      overlaps(maxw, mw_bytes, ws, ws_need))
    return SKA_ERR_INVALID_VALUE;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (d->norm == SKA_NORM_TOKEN)
    return sa_forward_token(d, q, k, v, cu_seqlens, seqused, sketch, lse, mass, ws, ws_bytes, s);
  ProtoFwdLaunch L;
  int nk = 0, nv = 0;
  if (!plan_forward(d, mass != nullptr, &L, &nk, &nv)) return SKA_ERR_UNSUPPORTED;
  FwdWs w;
  fwd_ws_layout(d, L, &w);
  if (w.total > ws_bytes) return SKA_ERR_WORKSPACE_TOO_SMALL;
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  WsHeader* hdr = reinterpret_cast<WsHeader*>(wsb + w.hdr);
  int32_t* prefix = reinterpret_cast<int32_t*>(wsb + w.prefix);
  float* partial = reinterpret_cast<float*>(wsb + w.partial);
  float* mass_partial = reinterpret_cast<float*>(wsb + w.mass_partial);

  const void* qb = q;
  const void* kb = k;
  const void* vb = v;
  if (d->in_dtype == SKA_F32) {
    if (launch_cast_f32_bf16(static_cast<const float*>(q), wsb + w.qb, int64_t(qn), s) != cudaSuccess)
      return SKA_ERR_CUDA;
    if (launch_cast_f32_bf16(static_cast<const float*>(k), wsb + w.kb, int64_t(kvn), s) != cudaSuccess)
      return SKA_ERR_CUDA;
    if (launch_cast_f32_bf16(static_cast<const float*>(v), wsb + w.vb, int64_t(kvn), s) != cudaSuccess)
      return SKA_ERR_CUDA;
    qb = wsb + w.qb;
    kb = wsb + w.kb;
    vb = wsb + w.vb;
  }

  if (cudaError_t e_ = launch_schedule(cu_seqlens, seqused, B, H, L.num_clusters, prefix, hdr, s); e_ != cudaSuccess) { record_error("launch_schedule", e_); return SKA_ERR_CUDA; }
  if (T > 0) {
    CUtensorMap mQ, mK, mV;
    const uint64_t qrows = uint64_t(d->q_per_user ? B : 1) * H * kp;
    if (!encode_2d(&mQ, qb, D, qrows, D, 64, L.kc)) return SKA_ERR_CUDA;
    if (!encode_2d(&mK, kb, uint64_t(H) * D, T, uint64_t(H) * D, 64, kTileTokens)) return SKA_ERR_CUDA;
    if (!encode_2d(&mV, vb, uint64_t(H) * D, T, uint64_t(H) * D, 64, kTileTokens)) return SKA_ERR_CUDA;
    ProtoFwdParams p{};
    p.cu_seqlens = cu_seqlens;
    p.seqused = seqused;
    p.tile_prefix = prefix;
    p.hdr = hdr;
    p.partial = partial;
    p.lse = lse;
    p.mass_partial = mass ? mass_partial : nullptr;
    p.maxw = maxw;
    p.B = B;
    p.H = H;
    p.k = kp;
    p.total_tokens = static_cast<int>(T);
    p.q_per_user = d->q_per_user;
    p.nk_slots = nk;
    p.nv_entries = nv;
    p.scale_log2 = d->scale * 1.4426950408889634f;
    p.budget_ns = wait_budget();
    p.debug_flags = g_debug_flags.load(std::memory_order_relaxed);
    cudaError_t e;
    {
      TimedRegion tr(s);
      e = launch_proto_fwd(D, L, mQ, mK, mV, p, s);
    }
    if (e != cudaSuccess) {
      record_error("fused kernel launch", e);
      return SKA_ERR_CUDA;
    }
  }
  if (cudaError_t e_ = launch_proto_combine(prefix, hdr, partial, mass ? mass_partial : nullptr, B, H, kp, D, sketch,
                                            mass, renormalize, s);
      e_ != cudaSuccess) {
    record_error("launch_proto_combine", e_);
    return SKA_ERR_CUDA;
  }
  if ((lse || maxw) && T > 0) {
    if (cudaError_t e_ = launch_fill_padding_lse(cu_seqlens, seqused, B, H, T, lse, maxw, s); e_ != cudaSuccess) { record_error("launch_fill_padding_lse", e_); return SKA_ERR_CUDA; }
  }
  return SKA_OK;
}

ska_status sa_forward(const ska_sa_desc* d, const void* q, const void* k, const void* v, const int32_t* cu_seqlens,
                      const int32_t* seqused, float* sketch, float* lse, float* mass, void* ws, size_t ws_bytes,
                      void* stream) {
  return sa_forward_impl(d, q, k, v, cu_seqlens, seqused, sketch, lse, mass, nullptr, false, ws, ws_bytes, stream);
}

ska_status sa_forward_diag(const ska_sa_desc* d, const void* q, const void* k, const void* v,
                           const int32_t* cu_seqlens, const int32_t* seqused, float* sketch, float* lse, float* mass,
                           float* token_max_weight, int32_t renormalize, void* ws, size_t ws_bytes, void* stream) {
  return sa_forward_impl(d, q, k, v, cu_seqlens, seqused, sketch, lse, mass, token_max_weight, renormalize != 0, ws,
                         ws_bytes, stream);
}

ska_status sa_weight_histogram(const float* values, int64_t n, int32_t bins, int32_t* counts, void* stream) {
  if (n < 0 || bins < 1 || bins > 4096) return SKA_ERR_INVALID_VALUE;
  if (!counts || (n > 0 && !values)) return SKA_ERR_INVALID_VALUE;
  if ((reinterpret_cast<uintptr_t>(values) & 3u) || (reinterpret_cast<uintptr_t>(counts) & 3u))
    return SKA_ERR_INVALID_VALUE;
  if (overlaps(values, size_t(n) * 4, counts, size_t(bins) * 4)) return SKA_ERR_INVALID_VALUE;
  if (no_device()) return SKA_ERR_CUDA;
  if (cudaError_t e = launch_weight_histogram(values, n, bins, counts, static_cast<cudaStream_t>(stream));
      e != cudaSuccess) {
    record_error("weight histogram launch", e);
    return SKA_ERR_CUDA;
  }
  return SKA_OK;
}

// Workspace of sa_backward: header, tile prefix, the dQ partial slots of one launch (one chunk of
// prototypes), then, for PROTO over several chunks, delta_i [T, H].
struct BwdWs {
  size_t dqp, delta, total;
};

bool bwd_ws_layout(const ska_sa_desc* d, int sms, BwdWs* w) {
  const int kc = sa_bwd_chunk(d->head_dim, d->num_protos);
  if (kc <= 0 || sms <= 0) return false;
  size_t off = sizeof(WsHeader);
  w->dqp = off = align256(off + size_t(d->num_users + 1) * 4);
  off = align256(off + (size_t(d->num_users) * d->num_heads + sms) * kc * d->head_dim * 4);
  w->delta = off;
  if (d->norm == SKA_NORM_PROTO && kc < d->num_protos) off = align256(off + size_t(d->total_tokens) * d->num_heads * 4);
  w->total = off;
  return true;
}

size_t sa_backward_workspace_size(const ska_sa_desc* d) {
  if (check_sa_desc(d) != SKA_OK) return 0;
  if (d->in_dtype != SKA_BF16 || !sa_bwd_supported(d->head_dim, d->num_protos)) return 0;
  BwdWs w;
  return bwd_ws_layout(d, device_sm_count(), &w) ? w.total : 0;
}

ska_status sa_backward(const ska_sa_desc* d, const void* q, const void* k, const void* v, const int32_t* cu_seqlens,
                       const int32_t* seqused, const float* sketch, const float* lse, const void* dsketch, float* dq,
                       float* dk, float* dv, void* ws, size_t ws_bytes, void* stream) {
  ska_status st = check_sa_desc(d);
  if (st != SKA_OK) return st;
  if (d->in_dtype != SKA_BF16 || !sa_bwd_supported(d->head_dim, d->num_protos)) return SKA_ERR_UNSUPPORTED;
  const int B = d->num_users, H = d->num_heads, D = d->head_dim, kp = d->num_protos;
  const int64_t T = d->total_tokens;
  if (!q || !dq || !cu_seqlens || !ws || !lse) return SKA_ERR_INVALID_VALUE;
  if (B > 0 && !dsketch) return SKA_ERR_INVALID_VALUE;
  if (T > 0 && (!k || !v || !dk || !dv)) return SKA_ERR_INVALID_VALUE;
  if (d->norm == SKA_NORM_TOKEN && B > 0 && !sketch) return SKA_ERR_INVALID_VALUE;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(sketch) || !aligned16(lse) ||
      !aligned16(dsketch) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv) ||
      (reinterpret_cast<uintptr_t>(ws) & 255u) || (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) ||
      (reinterpret_cast<uintptr_t>(seqused) & 3u))
    return SKA_ERR_INVALID_VALUE;
  if (no_device()) return SKA_ERR_CUDA;
  const size_t need = sa_backward_workspace_size(d);
  if (need == 0) return SKA_ERR_UNSUPPORTED;
  if (ws_bytes < need) return SKA_ERR_WORKSPACE_TOO_SMALL;
  const size_t qn = size_t(d->q_per_user ? B : 1) * H * kp * D, kvn = size_t(T) * H * D;
  const size_t outs[3][2] = {{reinterpret_cast<uintptr_t>(dq), qn * 4}, {reinterpret_cast<uintptr_t>(dk), kvn * 4},
                             {reinterpret_cast<uintptr_t>(dv), kvn * 4}};
  const void* ins[7] = {q, k, v, sketch, lse, dsketch, ws};
  const size_t insz[7] = {qn * 2, kvn * 2, kvn * 2, size_t(B) * H * kp * D * 4,
                          (d->norm == SKA_NORM_PROTO ? size_t(T) : size_t(B) * kp) * H * 4,
                          size_t(B) * H * kp * D * 2, need};
  for (int o = 0; o < 3; ++o) {
    for (int i = 0; i < 7; ++i)
      if (overlaps(reinterpret_cast<void*>(outs[o][0]), outs[o][1], ins[i], insz[i])) return SKA_ERR_INVALID_VALUE;
    for (int o2 = o + 1; o2 < 3; ++o2)
      if (overlaps(reinterpret_cast<void*>(outs[o][0]), outs[o][1], reinterpret_cast<void*>(outs[o2][0]),
                   outs[o2][1]))
        return SKA_ERR_INVALID_VALUE;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (B == 0) return SKA_OK;
  const int sms = device_sm_count();
  BwdWs w;
  if (!bwd_ws_layout(d, sms, &w)) return SKA_ERR_UNSUPPORTED;
  const int kc = sa_bwd_chunk(D, kp);  // prototypes per launch
  const int nchunks = kp / kc;
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  WsHeader* hdr = reinterpret_cast<WsHeader*>(wsb);
  int32_t* prefix = reinterpret_cast<int32_t*>(wsb + sizeof(WsHeader));
  float* dqp = reinterpret_cast<float*>(wsb + w.dqp);
  if (cudaError_t e_ = launch_schedule(cu_seqlens, seqused, B, H, sms, prefix, hdr, s); e_ != cudaSuccess) { record_error("launch_schedule", e_); return SKA_ERR_CUDA; }
  SaBwdParams p{};
  p.norm = d->norm;
  p.cu_seqlens = cu_seqlens;
  p.seqused = seqused;
  p.tile_prefix = prefix;
  p.hdr = hdr;
  p.lse = lse;
  p.sketch = sketch;
  p.dsketch = static_cast<const __nv_bfloat16*>(dsketch);
  p.dk = dk;
  p.dv = dv;
  p.dq_partial = dqp;
  p.B = B;
  p.H = H;
  p.k = kc;
  SaBwdChunk ck{};
  ck.delta = (d->norm == SKA_NORM_PROTO && nchunks > 1) ? reinterpret_cast<float*>(wsb + w.delta) : nullptr;
  ck.kt = kp;
  ck.j0 = 0;
  ck.pass = 0;
  ck.accumulate = 0;
  p.total_tokens = static_cast<int>(T);
  p.q_per_user = d->q_per_user;
  p.scale = d->scale;
  p.budget_ns = wait_budget();
  if (T == 0) {  // no tiles: the reduction writes zeros
    for (int c = 0; c < nchunks; ++c) {
      ck.j0 = c * kc;
      if (cudaError_t e_ = launch_sa_bwd_finish(p, ck, D, dq, s); e_ != cudaSuccess) { record_error("launch_sa_bwd_finish", e_); return SKA_ERR_CUDA; }
    }
    return SKA_OK;
  }
  CUtensorMap mQ, mDO, mK, mV;
  const uint64_t qrows = uint64_t(d->q_per_user ? B : 1) * H * kp;
  if (!encode_2d(&mQ, q, D, qrows, D, 64, kc)) return SKA_ERR_CUDA;
  if (!encode_2d(&mDO, dsketch, D, uint64_t(B) * H * kp, D, 64, kc)) return SKA_ERR_CUDA;
  if (!encode_2d(&mK, k, uint64_t(H) * D, T, uint64_t(H) * D, 64, 128)) return SKA_ERR_CUDA;
  if (!encode_2d(&mV, v, uint64_t(H) * D, T, uint64_t(H) * D, 64, 128)) return SKA_ERR_CUDA;
  if (nchunks == 1) {
    cudaError_t e;
    {
      TimedRegion tr(s);
      e = launch_sa_bwd(D, sms, mQ, mDO, mK, mV, p, ck, s);
    }
    if (e != cudaSuccess) {
      record_error("fused kernel launch", e);
      return SKA_ERR_CUDA;
    }
    if (cudaError_t e_ = launch_sa_bwd_finish(p, ck, D, dq, s); e_ != cudaSuccess) { record_error("launch_sa_bwd_finish", e_); return SKA_ERR_CUDA; }
    return SKA_OK;
  }
  // More prototypes than one CTA holds (the timed region spans every launch): PROTO first sums
  // delta_i = sum_j A_ij dA_ij over the chunks, one pass each; then every chunk forms its
  // gradients (with that delta_i in PROTO). dK and dV are summed over the chunks in chunk order,
  // and each chunk's dQ is reduced before the next chunk reuses the partial slots.
  TimedRegion tr(s);
  if (ck.delta) {
    ck.pass = 1;
    for (int c = 0; c < nchunks; ++c) {
      ck.j0 = c * kc;
      if (cudaError_t e = launch_sa_bwd(D, sms, mQ, mDO, mK, mV, p, ck, s); e != cudaSuccess) {
        record_error("fused kernel launch (delta)", e);
        return SKA_ERR_CUDA;
      }
    }
    ck.pass = 2;
  }
  for (int c = 0; c < nchunks; ++c) {
    ck.j0 = c * kc;
    ck.accumulate = c > 0;
    if (cudaError_t e = launch_sa_bwd(D, sms, mQ, mDO, mK, mV, p, ck, s); e != cudaSuccess) {
      record_error("fused kernel launch", e);
      return SKA_ERR_CUDA;
    }
    if (cudaError_t e_ = launch_sa_bwd_finish(p, ck, D, dq, s); e_ != cudaSuccess) { record_error("launch_sa_bwd_finish", e_); return SKA_ERR_CUDA; }
  }
  return SKA_OK;
}

size_t stca_forward_workspace_size(const ska_stca_desc* d) {
  if (check_stca_desc(d) != SKA_OK) return 0;
  FaWs w;
  int c, nk, nv;
  size_t sm;
  return stca_ws_size(d, &w, &c, &sm, &nk, &nv);
}

ska_status stca_forward(const ska_stca_desc* d, const void* q, const int32_t* cu_targets, const void* k_hist,
                        const void* v_hist, const int32_t* cu_hist, const int32_t* target_kv_len, const void* k_sk,
                        const void* v_sk, float* out, float* lse, void* ws, size_t ws_bytes, void* stream) {
  ska_status st = check_stca_desc(d);
  if (st != SKA_OK) return st;
  const int B = d->num_users, H = d->num_heads, D = d->head_dim, ks = d->num_sketch;
  const int64_t Tq = d->total_targets, Th = d->total_hist;
  if (B == 0 || Tq == 0) return SKA_OK;
  if (!q || !cu_targets || !cu_hist || !out || !ws) return SKA_ERR_INVALID_VALUE;
  if (Th > 0 && (!k_hist || !v_hist)) return SKA_ERR_INVALID_VALUE;
  if (ks > 0 && (!k_sk || !v_sk)) return SKA_ERR_INVALID_VALUE;
  if (!aligned16(q) || !aligned16(k_hist) || !aligned16(v_hist) || !aligned16(k_sk) || !aligned16(v_sk) ||
      !aligned16(out) || !aligned16(lse) || (reinterpret_cast<uintptr_t>(ws) & 255u) ||
      (reinterpret_cast<uintptr_t>(cu_targets) & 3u) || (reinterpret_cast<uintptr_t>(cu_hist) & 3u) ||
      (reinterpret_cast<uintptr_t>(target_kv_len) & 3u))
    return SKA_ERR_INVALID_VALUE;
  if (no_device()) return SKA_ERR_CUDA;
  FaWs w;
  int ctas, nk, nv;
  size_t smem;
  if (stca_ws_size(d, &w, &ctas, &smem, &nk, &nv) == 0) return SKA_ERR_UNSUPPORTED;
  if (ws_bytes < w.total) return SKA_ERR_WORKSPACE_TOO_SMALL;
  const size_t out_bytes = size_t(Tq) * H * D * 4, lse_bytes = size_t(Tq) * H * 4;
  const size_t qb_ = size_t(Tq) * H * D * 2, hb = size_t(Th) * H * D * 2, sb = size_t(B) * H * ks * D * 2;
  const void* ins[5] = {q, k_hist, v_hist, k_sk, v_sk};
  const size_t insz[5] = {qb_, hb, hb, sb, sb};
  for (int i = 0; i < 5; ++i)
    if (overlaps(out, out_bytes, ins[i], insz[i]) || overlaps(lse, lse_bytes, ins[i], insz[i]) ||
        overlaps(ws, w.total, ins[i], insz[i]))
      return SKA_ERR_INVALID_VALUE;
  if (overlaps(out, out_bytes, lse, lse_bytes) || overlaps(ws, w.total, out, out_bytes) ||
      overlaps(ws, w.total, lse, lse_bytes))
    return SKA_ERR_INVALID_VALUE;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  FaFwdParams p{};
  p.mode = 1;
  p.cu_keys = cu_hist;
  p.seqused = nullptr;
  p.cu_q = cu_targets;
  p.kv_len = target_kv_len;
  p.tile_prefix = reinterpret_cast<int32_t*>(wsb + w.tile_prefix);
  p.group = stca_group(d);
  p.hdr = reinterpret_cast<WsHeader*>(wsb + w.hdr);
  p.part_o = reinterpret_cast<float*>(wsb + w.part_o);
  p.part_ml = reinterpret_cast<float*>(wsb + w.part_ml);
  p.B = B;
  p.H = H;
  p.k = 0;
  p.ks = ks;
  p.q_per_user = 0;
  p.nk_slots = nk;
  p.nv_entries = nv;
  p.scale_log2 = d->scale * 1.4426950408889634f;
  p.budget_ns = wait_budget();
  p.debug_flags = g_debug_flags.load(std::memory_order_relaxed);
  if (cudaError_t e_ = launch_fa_schedule(p, ctas, s); e_ != cudaSuccess) { record_error("launch_fa_schedule", e_); return SKA_ERR_CUDA; }
  CUtensorMap mQ, mK, mV, mKs, mVs;
  if (!encode_2d(&mQ, q, uint64_t(H) * D, Tq, uint64_t(H) * D, 64, 128)) return SKA_ERR_CUDA;
  // maps over absent segments point at q with one row; no tile of theirs is ever loaded
  if (Th > 0) {
    if (!encode_2d(&mK, k_hist, uint64_t(H) * D, Th, uint64_t(H) * D, 64, 128)) return SKA_ERR_CUDA;
    if (!encode_2d(&mV, v_hist, uint64_t(H) * D, Th, uint64_t(H) * D, 64, 128)) return SKA_ERR_CUDA;
  } else {
    mK = mQ;
    mV = mQ;
  }
  if (ks > 0) {
    const uint64_t rows = uint64_t(B) * H * ks;
    if (!encode_2d(&mKs, k_sk, D, rows, D, 64, 128)) return SKA_ERR_CUDA;
    if (!encode_2d(&mVs, v_sk, D, rows, D, 64, 128)) return SKA_ERR_CUDA;
  } else {
    mKs = mQ;
    mVs = mQ;
  }
  cudaError_t e;
  {
    TimedRegion tr(s);
    e = launch_fa_fwd(D, ctas, smem, mQ, mK, mV, mKs, mVs, p, s);
  }
  if (e != cudaSuccess) {
    record_error("fused kernel launch", e);
    return SKA_ERR_CUDA;
  }
  if (cudaError_t e_ = launch_fa_combine(p, D, B * H * p.group, out, lse, nullptr, s); e_ != cudaSuccess) { record_error("launch_fa_combine", e_); return SKA_ERR_CUDA; }
  return SKA_OK;
}

size_t stca_backward_workspace_size(const ska_stca_desc* d) {
  if (check_stca_desc(d) != SKA_OK) return 0;
  size_t off = sizeof(WsHeader);
  off = align256(off + size_t(d->num_users + 1) * 4);
  off = align256(off + size_t(d->num_users + 1) * 4);
  off = align256(off + size_t(d->total_targets) * d->num_heads * 4);
  return off;
}

ska_status stca_backward(const ska_stca_desc* d, const void* q, const int32_t* cu_targets, const void* k_hist,
                         const void* v_hist, const int32_t* cu_hist, const int32_t* target_kv_len, const void* k_sk,
                         const void* v_sk, const float* out, const float* lse, const void* dout, float* dq,
                         float* dk_hist, float* dv_hist, float* dk_sk, float* dv_sk, void* ws, size_t ws_bytes,
                         void* stream) {
  ska_status st = check_stca_desc(d);
  if (st != SKA_OK) return st;
  const int B = d->num_users, H = d->num_heads, D = d->head_dim, ks = d->num_sketch;
  const int64_t Tq = d->total_targets, Th = d->total_hist;
  if (!stca_bwd_supported(D)) return SKA_ERR_UNSUPPORTED;
  if (B == 0) return SKA_OK;
  if (!cu_targets || !cu_hist || !ws) return SKA_ERR_INVALID_VALUE;
  if (Tq > 0 && (!q || !out || !lse || !dout || !dq)) return SKA_ERR_INVALID_VALUE;
  if (Th > 0 && (!k_hist || !v_hist || !dk_hist || !dv_hist)) return SKA_ERR_INVALID_VALUE;
  if (ks > 0 && (!k_sk || !v_sk || !dk_sk || !dv_sk)) return SKA_ERR_INVALID_VALUE;
  const void* al[13] = {q, k_hist, v_hist, k_sk, v_sk, out, lse, dout, dq, dk_hist, dv_hist, dk_sk, dv_sk};
  for (int i = 0; i < 13; ++i)
    if (!aligned16(al[i])) return SKA_ERR_INVALID_VALUE;
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) || (reinterpret_cast<uintptr_t>(cu_targets) & 3u) ||
      (reinterpret_cast<uintptr_t>(cu_hist) & 3u) || (reinterpret_cast<uintptr_t>(target_kv_len) & 3u))
    return SKA_ERR_INVALID_VALUE;
  const size_t need = stca_backward_workspace_size(d);
  if (ws_bytes < need) return SKA_ERR_WORKSPACE_TOO_SMALL;
  const size_t qb = size_t(Tq) * H * D * 2, hb = size_t(Th) * H * D * 2, sb = size_t(B) * H * ks * D * 2;
  const void* ins[8] = {q, k_hist, v_hist, k_sk, v_sk, out, lse, dout};
  const size_t insz[8] = {qb, hb, hb, sb, sb, qb * 2, size_t(Tq) * H * 4, qb};
  const void* outs[6] = {dq, dk_hist, dv_hist, dk_sk, dv_sk, ws};
  const size_t outsz[6] = {qb * 2, hb * 2, hb * 2, sb * 2, sb * 2, need};
  for (int o = 0; o < 6; ++o) {
    for (int i = 0; i < 8; ++i)
      if (overlaps(outs[o], outsz[o], ins[i], insz[i])) return SKA_ERR_INVALID_VALUE;
    for (int o2 = o + 1; o2 < 6; ++o2)
      if (overlaps(outs[o], outsz[o], outs[o2], outsz[o2])) return SKA_ERR_INVALID_VALUE;
  }
  if (no_device()) return SKA_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  StcaBwdParams p{};
  size_t off = sizeof(WsHeader);
  p.hdr = reinterpret_cast<WsHeader*>(wsb);
  p.kprefix = reinterpret_cast<int32_t*>(wsb + off);
  off = align256(off + size_t(B + 1) * 4);
  p.qprefix = reinterpret_cast<int32_t*>(wsb + off);
  off = align256(off + size_t(B + 1) * 4);
  p.delta = reinterpret_cast<float*>(wsb + off);
  p.cu_q = cu_targets;
  p.cu_k = cu_hist;
  p.kv_len = target_kv_len;
  p.lse = lse;
  p.dq = dq;
  p.dk_hist = dk_hist;
  p.dv_hist = dv_hist;
  p.dk_sk = dk_sk;
  p.dv_sk = dv_sk;
  p.B = B;
  p.H = H;
  p.ks = ks;
  p.scale = d->scale;
  p.budget_ns = wait_budget();
  if (cudaError_t e = launch_stca_bwd_prep(p, dout, out, Tq * H, D, s); e != cudaSuccess) {
    record_error("launch_stca_bwd_prep", e);
    return SKA_ERR_CUDA;
  }
  // maps over absent tensors point at the workspace's first row and are never loaded
  const void* dummy = Tq > 0 ? q : ws;
  CUtensorMap maps[6];
  const uint64_t qrows = std::max<int64_t>(Tq, 1), hrows = std::max<int64_t>(Th, 1);
  if (!encode_2d(&maps[0], Tq > 0 ? q : dummy, uint64_t(H) * D, qrows, uint64_t(H) * D, 64, 128)) return SKA_ERR_CUDA;
  if (!encode_2d(&maps[1], Tq > 0 ? dout : dummy, uint64_t(H) * D, qrows, uint64_t(H) * D, 64, 128)) return SKA_ERR_CUDA;
  if (!encode_2d(&maps[2], Th > 0 ? k_hist : dummy, uint64_t(H) * D, hrows, uint64_t(H) * D, 64, 128)) return SKA_ERR_CUDA;
  if (!encode_2d(&maps[3], Th > 0 ? v_hist : dummy, uint64_t(H) * D, hrows, uint64_t(H) * D, 64, 128)) return SKA_ERR_CUDA;
  const uint64_t srows = std::max<int64_t>(int64_t(B) * H * ks, 1);
  if (!encode_2d(&maps[4], ks > 0 ? k_sk : dummy, D, srows, D, 64, 128)) return SKA_ERR_CUDA;
  if (!encode_2d(&maps[5], ks > 0 ? v_sk : dummy, D, srows, D, 64, 128)) return SKA_ERR_CUDA;
  const int sms = device_sm_count();
  cudaError_t e;
  {
    TimedRegion tr(s);
    e = launch_stca_bwd(D, sms, sms, maps, p, s);
  }
  if (e == cudaSuccess) e = launch_stca_bwd_poison(p, Tq * H * D, Th * H * D, int64_t(B) * H * ks * D, s);
  if (e != cudaSuccess) {
    record_error("STCA backward launch", e);
    return SKA_ERR_CUDA;
  }
  return SKA_OK;
}

size_t sa_refine_workspace_size(const ska_refine_desc* d) {
  if (check_refine_desc(d) != SKA_OK) return 0;
  return sizeof(WsHeader);
}

ska_status sa_refine(const ska_refine_desc* d, const float* x_tilde, const float* x_hat, const void* w1,
                     const void* wg, const void* w2, const float* gamma1, const float* beta1, const float* gamma2,
                     const float* beta2, const void* w_q_next, float* x_next, float* x_bar, void* x_next_bf16,
                     void* q_next, void* ws, size_t ws_bytes, void* stream) {
  ska_status st = check_refine_desc(d);
  if (st != SKA_OK) return st;
  const int B = d->num_users, H = d->num_heads, k = d->num_protos, D = d->head_dim, F = d->ffn_dim;
  if (B == 0) return SKA_OK;
  if (!x_tilde || !x_hat || !w1 || !wg || !w2 || !x_next || !ws) return SKA_ERR_INVALID_VALUE;
  if ((w_q_next == nullptr) != (q_next == nullptr)) return SKA_ERR_INVALID_VALUE;
  const void* al[14] = {x_tilde, x_hat, w1, wg, w2, gamma1, beta1, gamma2, beta2, w_q_next, x_next, x_bar,
                        x_next_bf16, q_next};
  for (int i = 0; i < 14; ++i)
    if (!aligned16(al[i])) return SKA_ERR_INVALID_VALUE;
  if (reinterpret_cast<uintptr_t>(ws) & 255u) return SKA_ERR_INVALID_VALUE;
  if (ws_bytes < sizeof(WsHeader)) return SKA_ERR_WORKSPACE_TOO_SMALL;
  const size_t xb = size_t(B) * H * k * D * 4, wb = size_t(H) * D * F * 2, vb = size_t(H) * D * 4;
  const size_t xtb = d->x_tilde_shared ? size_t(H) * k * D * 4 : xb;
  const void* ins[10] = {x_tilde, x_hat, w1, wg, w2, gamma1, beta1, gamma2, beta2, w_q_next};
  const size_t insz[10] = {xtb, xb, wb, wb, wb, vb, vb, vb, vb, size_t(H) * D * D * 2};
  const void* outs[5] = {x_next, x_bar, x_next_bf16, q_next, ws};
  const size_t outsz[5] = {xb, xb, xb / 2, xb / 2, sizeof(WsHeader)};
  for (int o = 0; o < 5; ++o) {
    for (int i = 0; i < 10; ++i)
      if (overlaps(outs[o], outsz[o], ins[i], insz[i])) return SKA_ERR_INVALID_VALUE;
    for (int o2 = o + 1; o2 < 5; ++o2)
      if (overlaps(outs[o], outsz[o], outs[o2], outsz[o2])) return SKA_ERR_INVALID_VALUE;
  }
  if (no_device()) return SKA_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  WsHeader* hdr = static_cast<WsHeader*>(ws);
  if (cudaError_t e = cudaMemsetAsync(&hdr->status, 0, sizeof(int32_t), s); e != cudaSuccess) {
    record_error("cudaMemsetAsync(status)", e);
    return SKA_ERR_CUDA;
  }
  // W_1, W_g: [H d rows, F] in boxes of 64 columns x d rows; W_2: [H F rows, d] in 64 x F boxes;
  // W_Q: [H d rows, d] in 64 x d boxes
  CUtensorMap m1, mg, m2, mq;
  if (!encode_2d(&m1, w1, F, uint64_t(H) * D, F, 64, D)) return SKA_ERR_CUDA;
  if (!encode_2d(&mg, wg, F, uint64_t(H) * D, F, 64, D)) return SKA_ERR_CUDA;
  if (!encode_2d(&m2, w2, D, uint64_t(H) * F, D, 64, F)) return SKA_ERR_CUDA;
  if (w_q_next) {
    if (!encode_2d(&mq, w_q_next, D, uint64_t(H) * D, D, 64, D)) return SKA_ERR_CUDA;
  } else {
    mq = m1;  // never read
  }
  RefineParams p{};
  p.x_tilde = x_tilde;
  p.x_hat = x_hat;
  p.gamma1 = gamma1;
  p.beta1 = beta1;
  p.gamma2 = gamma2;
  p.beta2 = beta2;
  p.x_bar = x_bar;
  p.x_next = x_next;
  p.x_next_bf16 = static_cast<uint8_t*>(x_next_bf16);
  p.q_next = static_cast<uint8_t*>(q_next);
  p.status = &hdr->status;
  p.B = B;
  p.H = H;
  p.k = k;
  p.x_tilde_shared = d->x_tilde_shared ? 1 : 0;
  p.mode = 0;
  p.eps = d->eps;
  p.budget_ns = wait_budget();
  p.debug_flags = g_debug_flags.load(std::memory_order_relaxed);
  const int64_t tiles = int64_t(B) * H * ((k + 127) / 128);
  const int ctas = static_cast<int>(std::min<int64_t>(tiles, device_sm_count()));
  cudaError_t e;
  {
    TimedRegion tr(s);
    e = launch_sa_refine(D, F, ctas, m1, mg, m2, mq, p, s);
  }
  if (e == cudaSuccess) e = launch_refine_poison(D, p, s);
  if (e != cudaSuccess) {
    record_error("refinement kernel launch", e);
    return SKA_ERR_CUDA;
  }
  return SKA_OK;
}

ska_status sa_project_queries(int32_t num_users, int32_t num_heads, int32_t num_rows, int32_t head_dim,
                              const float* x, const void* w_q, void* q_out, void* ws, size_t ws_bytes,
                              void* stream) {
  if (num_users < 0 || num_heads < 1 || num_rows < 1) return SKA_ERR_INVALID_VALUE;
  if (!sa_refine_supported(head_dim, 2 * head_dim)) return SKA_ERR_UNSUPPORTED;
  const int B = num_users, H = num_heads, k = num_rows, D = head_dim;
  if (int64_t(B) * H * k * D >= (int64_t(1) << 31)) return SKA_ERR_INVALID_VALUE;
  if (B == 0) return SKA_OK;
  if (!x || !w_q || !q_out || !ws) return SKA_ERR_INVALID_VALUE;
  if (!aligned16(x) || !aligned16(w_q) || !aligned16(q_out) || (reinterpret_cast<uintptr_t>(ws) & 255u))
    return SKA_ERR_INVALID_VALUE;
  if (ws_bytes < sizeof(WsHeader)) return SKA_ERR_WORKSPACE_TOO_SMALL;
  const size_t xb = size_t(B) * H * k * D * 4, qb = xb / 2, wqb = size_t(H) * D * D * 2;
  if (overlaps(q_out, qb, x, xb) || overlaps(q_out, qb, w_q, wqb) || overlaps(ws, sizeof(WsHeader), x, xb) ||
      overlaps(ws, sizeof(WsHeader), w_q, wqb) || overlaps(ws, sizeof(WsHeader), q_out, qb))
    return SKA_ERR_INVALID_VALUE;
  if (no_device()) return SKA_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  WsHeader* hdr = static_cast<WsHeader*>(ws);
  if (cudaError_t e = cudaMemsetAsync(&hdr->status, 0, sizeof(int32_t), s); e != cudaSuccess) {
    record_error("cudaMemsetAsync(status)", e);
    return SKA_ERR_CUDA;
  }
  CUtensorMap mq;
  if (!encode_2d(&mq, w_q, D, uint64_t(H) * D, D, 64, D)) return SKA_ERR_CUDA;
  RefineParams p{};
  p.x_tilde = x;
  p.q_next = static_cast<uint8_t*>(q_out);
  p.status = &hdr->status;
  p.B = B;
  p.H = H;
  p.k = k;
  p.mode = 1;
  p.eps = 1.f;
  p.budget_ns = wait_budget();
  p.debug_flags = g_debug_flags.load(std::memory_order_relaxed);
  const int64_t tiles = int64_t(B) * H * ((k + 127) / 128);
  const int ctas = static_cast<int>(std::min<int64_t>(tiles, device_sm_count()));
  cudaError_t e = launch_sa_refine(D, 2 * D, ctas, mq, mq, mq, mq, p, s);
  if (e == cudaSuccess) e = launch_refine_poison(D, p, s);
  if (e != cudaSuccess) {
    record_error("projection kernel launch", e);
    return SKA_ERR_CUDA;
  }
  return SKA_OK;
}

size_t sa_cache_bytes(const ska_cache_desc* d) { return cache_desc_ok(d) ? cache_bytes(*d) : 0; }

ska_status sa_cache_init(const ska_cache_desc* d, void* cache, size_t nbytes, void* stream) {
  if (!cache_desc_ok(d)) return SKA_ERR_INVALID_VALUE;
  if (!cache || (reinterpret_cast<uintptr_t>(cache) & 255u)) return SKA_ERR_INVALID_VALUE;
  if (nbytes < cache_bytes(*d)) return SKA_ERR_WORKSPACE_TOO_SMALL;
  if (no_device()) return SKA_ERR_CUDA;
  if (cudaError_t e = launch_cache_init(*d, cache, static_cast<cudaStream_t>(stream)); e != cudaSuccess) {
    record_error("cache init launch", e);
    return SKA_ERR_CUDA;
  }
  return SKA_OK;
}

ska_status sa_cache_put(const ska_cache_desc* d, void* cache, size_t nbytes, const ska_cache_key* keys,
                        const float* rows, int32_t n, int64_t now, int32_t* slots, void* stream) {
  if (!cache_desc_ok(d) || n < 0) return SKA_ERR_INVALID_VALUE;
  if (!cache || (reinterpret_cast<uintptr_t>(cache) & 255u)) return SKA_ERR_INVALID_VALUE;
  if (nbytes < cache_bytes(*d)) return SKA_ERR_WORKSPACE_TOO_SMALL;
  if (n == 0) return SKA_OK;
  if (!keys || !rows || !slots || !aligned16(rows) || (reinterpret_cast<uintptr_t>(keys) & 7u) ||
      (reinterpret_cast<uintptr_t>(slots) & 3u))
    return SKA_ERR_INVALID_VALUE;
  const size_t cb = cache_bytes(*d), rb = size_t(n) * d->row_floats * 4;
  if (overlaps(cache, cb, keys, size_t(n) * sizeof(ska_cache_key)) || overlaps(cache, cb, rows, rb) ||
      overlaps(cache, cb, slots, size_t(n) * 4) || overlaps(slots, size_t(n) * 4, rows, rb) ||
      overlaps(slots, size_t(n) * 4, keys, size_t(n) * sizeof(ska_cache_key)))
    return SKA_ERR_INVALID_VALUE;
  if (no_device()) return SKA_ERR_CUDA;
  if (cudaError_t e = launch_cache_put(*d, cache, keys, rows, n, now, slots, static_cast<cudaStream_t>(stream));
      e != cudaSuccess) {
    record_error("cache put launch", e);
    return SKA_ERR_CUDA;
  }
  return SKA_OK;
}

ska_status sa_cache_get(const ska_cache_desc* d, const void* cache, size_t nbytes, const ska_cache_key* keys,
                        int32_t n, int64_t now, float* out, int32_t* hits, void* stream) {
  if (!cache_desc_ok(d) || n < 0) return SKA_ERR_INVALID_VALUE;
  if (!cache || (reinterpret_cast<uintptr_t>(cache) & 255u)) return SKA_ERR_INVALID_VALUE;
  if (nbytes < cache_bytes(*d)) return SKA_ERR_WORKSPACE_TOO_SMALL;
  if (n == 0) return SKA_OK;
  if (!keys || !out || !hits || !aligned16(out) || (reinterpret_cast<uintptr_t>(keys) & 7u) ||
      (reinterpret_cast<uintptr_t>(hits) & 3u))
    return SKA_ERR_INVALID_VALUE;
  const size_t cb = cache_bytes(*d), ob = size_t(n) * d->row_floats * 4;
  if (overlaps(out, ob, cache, cb) || overlaps(out, ob, keys, size_t(n) * sizeof(ska_cache_key)) ||
      overlaps(hits, size_t(n) * 4, cache, cb) || overlaps(hits, size_t(n) * 4, out, ob) ||
      overlaps(hits, size_t(n) * 4, keys, size_t(n) * sizeof(ska_cache_key)))
    return SKA_ERR_INVALID_VALUE;
  if (no_device()) return SKA_ERR_CUDA;
  if (cudaError_t e = launch_cache_get(*d, cache, keys, n, now, out, hits, static_cast<cudaStream_t>(stream));
      e != cudaSuccess) {
    record_error("cache get launch", e);
    return SKA_ERR_CUDA;
  }
  return SKA_OK;
}

}  // extern "C"
