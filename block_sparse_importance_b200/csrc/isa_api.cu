// C ABI of libisa.so (declared in include/isa.h): argument checks, the
// per-context device status word, workspace carving and kernel launches.
// The library allocates no device memory in a call path; every device buffer
// belongs to the caller.  (isa_pipeline_host creates two copy streams on its
// first call, kept by the context, and a few events per call.)

#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "isa.h"
#include "isa_internal.h"

struct isa_context {
  int device;
  int num_sms;
  int* d_status;
  uint64_t wait_timeout_ns;  // 0: the kernels' default
  int stall_attention;       // failure-detection test hook
  cudaStream_t copy_in, copy_out;  // isa_pipeline_host's copy streams (made on first use)
  char last_error[512];
};

namespace {

using namespace isa_impl;

isa_status fail(isa_context* ctx, isa_status s, const char* fmt, ...) {
  if (ctx) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(ctx->last_error, sizeof(ctx->last_error), fmt, ap);
    va_end(ap);
  }
  return s;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t round_up(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Makes the context's device current for the duration of a call.
class DeviceGuard {
 public:
  explicit DeviceGuard(int dev) {
    ok_ = cudaGetDevice(&prev_) == cudaSuccess;
    if (ok_ && prev_ != dev) ok_ = cudaSetDevice(dev) == cudaSuccess;
    restore_ = ok_ && prev_ != dev;
  }
  ~DeviceGuard() {
    if (restore_) cudaSetDevice(prev_);
  }
  bool ok() const { return ok_; }

 private:
  int prev_ = 0;
  bool ok_ = false, restore_ = false;
};

int nblocks(const isa_shape* s) { return (s->seq_len + s->k_block - 1) / s->k_block; }

isa_status check_shape(isa_context* ctx, const isa_shape* s) {
  if (!ctx) return ISA_ERR_INVALID_ARG;
  ctx->last_error[0] = 0;
  if (!s) return fail(ctx, ISA_ERR_INVALID_ARG, "shape is NULL");
  if (s->batch < 1 || s->heads < 1 || s->seq_len < 1)
    return fail(ctx, ISA_ERR_INVALID_ARG, "batch, heads and seq_len must be >= 1");
  if (s->head_dim != 64 && s->head_dim != 128)
    return fail(ctx, ISA_ERR_UNSUPPORTED, "head_dim %d: only 64 and 128 are built", s->head_dim);
  if (s->k_block != 16 && s->k_block != 32 && s->k_block != 64 && s->k_block != 128)
    return fail(ctx, ISA_ERR_INVALID_ARG, "k_block %d: must be 16, 32, 64 or 128", s->k_block);
  if (s->num_groups < 1) return fail(ctx, ISA_ERR_INVALID_ARG, "num_groups must be >= 1");
  if (!s->q_offsets) {
    if (s->q_block < 1) return fail(ctx, ISA_ERR_INVALID_ARG, "q_block must be >= 1");
    const long long g = (static_cast<long long>(s->seq_len) + s->q_block - 1) / s->q_block;
    if (g != s->num_groups)
      return fail(ctx, ISA_ERR_INVALID_ARG, "num_groups %d != ceil(seq_len / q_block) = %lld", s->num_groups, g);
  } else {
    if (!aligned(s->q_offsets, 4)) return fail(ctx, ISA_ERR_INVALID_ARG, "q_offsets not 4-byte aligned");
    if (s->num_groups > s->seq_len) return fail(ctx, ISA_ERR_INVALID_ARG, "more groups than rows");
  }
  if (!std::isfinite(s->scale) || !(s->scale > 0.0f))
    return fail(ctx, ISA_ERR_INVALID_ARG, "scale must be finite and > 0");
  const long long bh = static_cast<long long>(s->batch) * s->heads;
  if (bh * s->seq_len > (1LL << 40) || bh > (1LL << 30))
    return fail(ctx, ISA_ERR_INVALID_ARG, "tensor too large");
  return ISA_OK;
}

isa_status check_ptr(isa_context* ctx, const void* p, const char* name, size_t align) {
  if (!p) return fail(ctx, ISA_ERR_INVALID_ARG, "%s is NULL", name);
  if (!aligned(p, align)) return fail(ctx, ISA_ERR_INVALID_ARG, "%s is not %zu-byte aligned", name, align);
  return ISA_OK;
}

isa_status cuda_status(isa_context* ctx, int e, const char* what) {
  if (e == 0) return ISA_OK;
  if (e < 0) return fail(ctx, ISA_ERR_CUDA, "%s: tensor map encoding failed", what);
  return fail(ctx, ISA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(static_cast<cudaError_t>(e)));
}

#define ISA_TRY(x)                  \
  do {                              \
    const isa_status s_ = (x);      \
    if (s_ != ISA_OK) return s_;    \
  } while (0)

// Shapes of the token-clustering calls: only batch, heads, seq_len and
// head_dim are read.
isa_status check_rows_shape(isa_context* ctx, const isa_shape* s) {
  if (!ctx) return ISA_ERR_INVALID_ARG;
  ctx->last_error[0] = 0;
  if (!s) return fail(ctx, ISA_ERR_INVALID_ARG, "shape is NULL");
  if (s->batch < 1 || s->heads < 1 || s->seq_len < 1)
    return fail(ctx, ISA_ERR_INVALID_ARG, "batch, heads and seq_len must be >= 1");
  if (s->head_dim != 64 && s->head_dim != 128)
    return fail(ctx, ISA_ERR_UNSUPPORTED, "head_dim %d: only 64 and 128 are built", s->head_dim);
  const long long bh = static_cast<long long>(s->batch) * s->heads;
  if (bh * s->seq_len > (1LL << 31) - 1 || bh > 65535)
    return fail(ctx, ISA_ERR_INVALID_ARG, "tensor too large for the clustering calls");
  return ISA_OK;
}

constexpr int kMaxClusters = 8192;

isa_status check_clusters(isa_context* ctx, const isa_shape* s, int32_t C) {
  if (C < 1 || C > s->seq_len || C > kMaxClusters)
    return fail(ctx, ISA_ERR_INVALID_ARG, "n_clusters = %d: need 1 <= n_clusters <= min(seq_len, %d)", C, kMaxClusters);
  return ISA_OK;
}

size_t cluster_ws(const isa_shape* s, int32_t C) {
  const size_t BH = static_cast<size_t>(s->batch) * s->heads;
  const size_t cp = static_cast<size_t>(cluster_cpad(C));
  return 2 * round_up(BH * cp * s->head_dim * 2) + round_up(BH * cp * 4);
}

ClusterLaunch cluster_launch(const isa_shape* s, int32_t C, const void* x, float* mu, void* ws) {
  ClusterLaunch l{};
  l.BH = s->batch * s->heads;
  l.N = s->seq_len;
  l.D = s->head_dim;
  l.C = C;
  l.Cpad = cluster_cpad(C);
  l.x = x;
  l.mu = mu;
  uint8_t* w = static_cast<uint8_t*>(ws);
  const size_t BH = static_cast<size_t>(l.BH);
  l.mu_hi = reinterpret_cast<uint16_t*>(w);
  w += round_up(BH * l.Cpad * l.D * 2);
  l.mu_lo = reinterpret_cast<uint16_t*>(w);
  w += round_up(BH * l.Cpad * l.D * 2);
  l.mu_nsq = reinterpret_cast<float*>(w);
  return l;
}

size_t attn_ws_bytes(const isa_shape* s) {
  const bool list = s->q_offsets != nullptr || s->q_block > 128;
  return list ? round_up(attn_list_workspace_bytes(s->seq_len, s->num_groups)) : 0;
}

isa_status do_score(isa_context* ctx, const isa_shape* s, const void* q, const void* k, int32_t C, int32_t iters,
                    float* mass, float* centroids, int32_t* counts, void* ws, size_t ws_bytes, cudaStream_t st) {
  ISA_TRY(check_ptr(ctx, q, "q", 16));
  ISA_TRY(check_ptr(ctx, k, "k", 16));
  ISA_TRY(check_ptr(ctx, mass, "mass", 16));
  if (C < 1 || C > 16) return fail(ctx, ISA_ERR_INVALID_ARG, "n_clusters %d: must be 1..16", C);
  if (iters < 1 || iters > 16) return fail(ctx, ISA_ERR_INVALID_ARG, "n_iters %d: must be 1..16", iters);
  if (centroids && !aligned(centroids, 16)) return fail(ctx, ISA_ERR_INVALID_ARG, "centroids not 16-byte aligned");
  if (counts && !aligned(counts, 4)) return fail(ctx, ISA_ERR_INVALID_ARG, "counts not 4-byte aligned");
  const size_t need = score_workspace_bytes(s->batch, s->heads, s->seq_len, s->head_dim, s->num_groups, s->k_block, C);
  if (!ws || ws_bytes < need)
    return fail(ctx, ISA_ERR_INVALID_ARG, "score workspace %zu bytes < %zu needed", ws_bytes, need);
  if (!aligned(ws, 256)) return fail(ctx, ISA_ERR_INVALID_ARG, "workspace not 256-byte aligned");
  const size_t BH = static_cast<size_t>(s->batch) * s->heads;
  const size_t nK = nblocks(s);
  char* w = static_cast<char*>(ws);
  ScoreLaunch l{};
  l.B = s->batch;
  l.H = s->heads;
  l.N = s->seq_len;
  l.D = s->head_dim;
  l.G = s->num_groups;
  l.Bk = s->k_block;
  l.q_block = s->q_block;
  l.C = C;
  l.iters = iters;
  l.q_offsets = s->q_offsets;
  l.scale = s->scale;
  l.q = q;
  l.k = k;
  l.mass = mass;
  l.kbar_hi = reinterpret_cast<uint16_t*>(w);
  l.kbar_lo = l.kbar_hi + BH * nK * s->head_dim;
  w += round_up(BH * nK * s->head_dim * 4);
  l.centroids = centroids ? centroids : reinterpret_cast<float*>(w);
  w += round_up(BH * s->num_groups * C * s->head_dim * 4);
  l.counts = counts ? counts : reinterpret_cast<int32_t*>(w);
  w += round_up(BH * s->num_groups * C * 4);
  l.kb_next = reinterpret_cast<uint32_t*>(w);
  l.status = ctx->d_status;
  l.num_sms = ctx->num_sms;
  return cuda_status(ctx, launch_score(l, st), "isa_score");
}

isa_status do_select(isa_context* ctx, const isa_shape* s, const float* mass, int32_t ne, int32_t ns, uint64_t seed,
                     int32_t* idx, float* log_w, cudaStream_t st, int h_base = 0, int b_base = 0,
                     const int32_t* ne_rows = nullptr, bool discard_mass = false) {
  ISA_TRY(check_ptr(ctx, mass, "mass", 4));
  ISA_TRY(check_ptr(ctx, idx, "idx", 4));
  ISA_TRY(check_ptr(ctx, log_w, "log_w", 4));
  const int nK = nblocks(s);
  if (ne < 0 || ns < 0 || ne + ns < 1 || ne + ns > nK)
    return fail(ctx, ISA_ERR_INVALID_ARG, "need 0 <= n_exact, n_sample and 1 <= n_exact + n_sample <= nK = %d", nK);
  if (nK > 16384) return fail(ctx, ISA_ERR_UNSUPPORTED, "nK = %d key blocks: at most 16384 are built", nK);
  SelectLaunch l{};
  l.B = s->batch;
  l.H = s->heads;
  l.G = s->num_groups;
  l.nK = nK;
  l.n_exact = ne;
  l.n_sample = ns;
  l.h_base = h_base;
  l.b_base = b_base;
  l.seed = seed;
  l.mass = mass;
  l.idx = idx;
  l.log_w = log_w;
  l.ne_rows = ne_rows;
  l.status = ctx->d_status;
  l.num_sms = ctx->num_sms;
  l.discard_mass = discard_mass ? 1 : 0;
  return cuda_status(ctx, launch_select(l, st), "isa_select");
}

isa_status do_attention(isa_context* ctx, const isa_shape* s, const void* q, const void* k, const void* v,
                        const int32_t* idx, const float* log_w, int32_t n_sel, void* out, float* lse, void* ws,
                        size_t ws_bytes, bool dense, cudaStream_t st) {
  ISA_TRY(check_ptr(ctx, q, "q", 16));
  ISA_TRY(check_ptr(ctx, k, "k", 16));
  ISA_TRY(check_ptr(ctx, v, "v", 16));
  ISA_TRY(check_ptr(ctx, out, "out", 16));
  if (lse && !aligned(lse, 4)) return fail(ctx, ISA_ERR_INVALID_ARG, "lse not 4-byte aligned");
  AttnLaunch l{};
  l.B = s->batch;
  l.H = s->heads;
  l.N = s->seq_len;
  l.D = s->head_dim;
  l.G = s->num_groups;
  l.Bk = s->k_block;
  l.q_block = s->q_block;
  l.q_offsets = s->q_offsets;
  l.out = out;
  l.lse = lse;
  l.scale = s->scale;
  l.status = ctx->d_status;
  l.num_sms = ctx->num_sms;
  l.wait_timeout_ns = ctx->wait_timeout_ns;
  l.stall = ctx->stall_attention;
  if (dense) {
    l.mode = kAttnDense;
    l.S = 1;
    l.G = 1;
  } else {
    ISA_TRY(check_ptr(ctx, idx, "idx", 4));
    ISA_TRY(check_ptr(ctx, log_w, "log_w", 4));
    if (n_sel < 1) return fail(ctx, ISA_ERR_INVALID_ARG, "n_sel must be >= 1");
    l.S = n_sel;
    l.idx = idx;
    l.log_w = log_w;
    const size_t need = attn_ws_bytes(s);
    if (need) {
      if (!ws || ws_bytes < need)
        return fail(ctx, ISA_ERR_INVALID_ARG, "attention workspace %zu bytes < %zu needed", ws_bytes, need);
      if (!aligned(ws, 16)) return fail(ctx, ISA_ERR_INVALID_ARG, "workspace not 16-byte aligned");
      l.mode = kAttnList;
      l.workspace = ws;
    } else {
      l.mode = kAttnGroups;
    }
  }
  return cuda_status(ctx, launch_attention(l, q, k, v, st), dense ? "isa_dense_attention" : "isa_attention");
}

size_t pipeline_bytes(const isa_shape* s, const isa_params* p) {
  const size_t rows = static_cast<size_t>(s->batch) * s->heads * s->num_groups;
  const size_t S = static_cast<size_t>(p->n_exact) + p->n_sample;
  return round_up(score_workspace_bytes(s->batch, s->heads, s->seq_len, s->head_dim, s->num_groups, s->k_block,
                                        p->n_clusters)) +
         round_up(rows * nblocks(s) * 4) + 2 * round_up(rows * S * 4) + attn_ws_bytes(s);
}

isa_status do_pipeline(isa_context* ctx, const isa_shape* s, const isa_params* p, const void* q, const void* k,
                       const void* v, void* out, float* lse, int32_t* plan_idx, float* plan_lw, void* ws,
                       size_t ws_bytes, cudaStream_t st, int h_base = 0, int b_base = 0) {
  if (!p) return fail(ctx, ISA_ERR_INVALID_ARG, "params is NULL");
  if (p->n_clusters < 1 || p->n_clusters > 16) return fail(ctx, ISA_ERR_INVALID_ARG, "n_clusters must be 1..16");
  const size_t need = pipeline_bytes(s, p);
  if (!ws || ws_bytes < need)
    return fail(ctx, ISA_ERR_INVALID_ARG, "pipeline workspace %zu bytes < %zu needed", ws_bytes, need);
  if (!aligned(ws, 256)) return fail(ctx, ISA_ERR_INVALID_ARG, "workspace not 256-byte aligned");
  const size_t rows = static_cast<size_t>(s->batch) * s->heads * s->num_groups;
  const size_t S = static_cast<size_t>(p->n_exact) + p->n_sample;
  char* w = static_cast<char*>(ws);
  const size_t score_ws = round_up(score_workspace_bytes(s->batch, s->heads, s->seq_len, s->head_dim, s->num_groups,
                                                         s->k_block, p->n_clusters));
  void* sws = w;
  w += score_ws;
  float* mass = reinterpret_cast<float*>(w);
  w += round_up(rows * nblocks(s) * 4);
  int32_t* idx = plan_idx ? plan_idx : reinterpret_cast<int32_t*>(w);
  w += round_up(rows * S * 4);
  float* lw = plan_lw ? plan_lw : reinterpret_cast<float*>(w);
  w += round_up(rows * S * 4);
  void* aws = w;
  ISA_TRY(do_score(ctx, s, q, k, p->n_clusters, p->n_iters, mass, nullptr, nullptr, sws, score_ws, st));
  ISA_TRY(do_select(ctx, s, mass, p->n_exact, p->n_sample, p->seed, idx, lw, st, h_base, b_base));
  return do_attention(ctx, s, q, k, v, idx, lw, static_cast<int32_t>(S), out, lse, aws, attn_ws_bytes(s), false, st);
}

// isa_plan: heads per chunk, so that one chunk's mass stays inside L2 (126 MB)
// between the mass kernel that writes it and the selector that reads it,
// while a chunk still gives the kernels enough CTAs to fill the SMs (at the
// Hunyuan shape one head's mass is 28 MB and fills under half the SMs).
constexpr size_t kPlanChunkMassBytes = size_t(88) << 20;

int plan_chunk_heads(const isa_shape* s) {
  const size_t per_head = static_cast<size_t>(s->num_groups) * nblocks(s) * 4;
  size_t hc = per_head ? kPlanChunkMassBytes / per_head : 1;
  if (hc < 1) hc = 1;
  const size_t H = s->heads > 0 ? static_cast<size_t>(s->heads) : 1;
  if (hc > H) hc = H;
  // the same number of chunks with the heads spread evenly over them, so that
  // no chunk is a small remainder that leaves most SMs idle
  const size_t chunks = (H + hc - 1) / hc;
  hc = (H + chunks - 1) / chunks;
  return static_cast<int>(hc);
}

size_t plan_bytes(const isa_shape* s, const isa_params* p) {
  const int hc = plan_chunk_heads(s);
  return round_up(score_workspace_bytes(1, hc, s->seq_len, s->head_dim, s->num_groups, s->k_block, p->n_clusters)) +
         round_up(static_cast<size_t>(hc) * s->num_groups * nblocks(s) * 4);
}

}  // namespace

extern "C" {

isa_status isa_create(int device, isa_context** out) {
  if (!out) return ISA_ERR_INVALID_ARG;
  *out = nullptr;
  int prev = 0;
  if (cudaGetDevice(&prev) != cudaSuccess) return ISA_ERR_CUDA;
  if (cudaSetDevice(device) != cudaSuccess) return ISA_ERR_CUDA;
  cudaDeviceProp prop;
  isa_status st = ISA_OK;
  int* d_status = nullptr;
  if (cudaGetDeviceProperties(&prop, device) != cudaSuccess) {
    st = ISA_ERR_CUDA;
  } else if (prop.major != 10 || prop.minor != 0) {
    st = ISA_ERR_UNSUPPORTED;  // the kernels are built for sm_100a only
  } else if (cudaMalloc(&d_status, sizeof(int)) != cudaSuccess || cudaMemset(d_status, 0, sizeof(int)) != cudaSuccess) {
    st = ISA_ERR_CUDA;
  }
  if (st == ISA_OK) {
    isa_context* c = new isa_context();
    c->device = device;
    c->num_sms = prop.multiProcessorCount;
    c->d_status = d_status;
    c->wait_timeout_ns = 0;
    c->stall_attention = 0;
    c->last_error[0] = 0;
    *out = c;
  } else if (d_status) {
    cudaFree(d_status);
  }
  cudaSetDevice(prev);
  return st;
}

void isa_destroy(isa_context* ctx) {
  if (!ctx) return;
  DeviceGuard g(ctx->device);
  cudaFree(ctx->d_status);
  if (ctx->copy_in) cudaStreamDestroy(ctx->copy_in);
  if (ctx->copy_out) cudaStreamDestroy(ctx->copy_out);
  delete ctx;
}

const char* isa_status_string(isa_status s) {
  switch (s) {
    case ISA_OK: return "ok";
    case ISA_ERR_INVALID_ARG: return "invalid argument";
    case ISA_ERR_UNSUPPORTED: return "unsupported";
    case ISA_ERR_CUDA: return "CUDA error";
    case ISA_ERR_TIMEOUT: return "device pipeline wait timed out";
    case ISA_ERR_DEVICE_CHECK: return "device-side check failed";
  }
  return "unknown status";
}

const char* isa_last_error(const isa_context* ctx) { return ctx ? ctx->last_error : "no context"; }

isa_status isa_sync_status(isa_context* ctx, void* stream) {
  if (!ctx) return ISA_ERR_INVALID_ARG;
  DeviceGuard g(ctx->device);
  if (!g.ok()) return fail(ctx, ISA_ERR_CUDA, "cannot select device %d", ctx->device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int h = 0;
  cudaError_t e = cudaMemcpyAsync(&h, ctx->d_status, sizeof(int), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e == cudaSuccess) e = cudaMemsetAsync(ctx->d_status, 0, sizeof(int), st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return fail(ctx, ISA_ERR_CUDA, "isa_sync_status: %s", cudaGetErrorString(e));
  if (h == ISA_ERR_TIMEOUT) return ISA_ERR_TIMEOUT;
  if (h != 0) return ISA_ERR_DEVICE_CHECK;
  return ISA_OK;
}

isa_status isa_debug_set(isa_context* ctx, int32_t knob, uint64_t value) {
  if (!ctx) return ISA_ERR_INVALID_ARG;
  switch (knob) {
    case ISA_DEBUG_WAIT_TIMEOUT_NS: ctx->wait_timeout_ns = value; return ISA_OK;
    case ISA_DEBUG_STALL_ATTENTION: ctx->stall_attention = value != 0; return ISA_OK;
  }
  return fail(ctx, ISA_ERR_INVALID_ARG, "isa_debug_set: unknown knob %d", knob);
}

size_t isa_score_workspace_bytes(const isa_shape* s, int32_t n_clusters) {
  if (!s || n_clusters < 1) return 0;
  return score_workspace_bytes(s->batch, s->heads, s->seq_len, s->head_dim, s->num_groups, s->k_block, n_clusters);
}

isa_status isa_score(isa_context* ctx, const isa_shape* shape, const void* q, const void* k, int32_t n_clusters,
                     int32_t n_iters, float* mass, float* centroids, int32_t* counts, void* workspace,
                     size_t workspace_bytes, void* stream) {
  ISA_TRY(check_shape(ctx, shape));
  DeviceGuard g(ctx->device);
  if (!g.ok()) return fail(ctx, ISA_ERR_CUDA, "cannot select device %d", ctx->device);
  return do_score(ctx, shape, q, k, n_clusters, n_iters, mass, centroids, counts, workspace, workspace_bytes,
                  static_cast<cudaStream_t>(stream));
}

isa_status isa_select(isa_context* ctx, const isa_shape* shape, const float* mass, int32_t n_exact, int32_t n_sample,
                      uint64_t seed, int32_t* idx, float* log_w, void* stream) {
  ISA_TRY(check_shape(ctx, shape));
  DeviceGuard g(ctx->device);
  if (!g.ok()) return fail(ctx, ISA_ERR_CUDA, "cannot select device %d", ctx->device);
  return do_select(ctx, shape, mass, n_exact, n_sample, seed, idx, log_w, static_cast<cudaStream_t>(stream));
}

isa_status isa_select_top_p(isa_context* ctx, const isa_shape* shape, const float* mass, double top_p,
                            int32_t n_select, uint64_t seed, int32_t* idx, float* log_w, int32_t* n_exact_rows,
                            void* stream) {
  ISA_TRY(check_shape(ctx, shape));
  DeviceGuard g(ctx->device);
  if (!g.ok()) return fail(ctx, ISA_ERR_CUDA, "cannot select device %d", ctx->device);
  ISA_TRY(check_ptr(ctx, mass, "mass", 4));
  ISA_TRY(check_ptr(ctx, idx, "idx", 4));
  ISA_TRY(check_ptr(ctx, log_w, "log_w", 4));
  ISA_TRY(check_ptr(ctx, n_exact_rows, "n_exact_rows", 4));
  if (!(top_p > 0.0) || top_p > 1.0) return fail(ctx, ISA_ERR_INVALID_ARG, "top_p = %g: need 0 < top_p <= 1", top_p);
  const int nK = nblocks(shape);
  if (n_select < 1 || n_select > nK)
    return fail(ctx, ISA_ERR_INVALID_ARG, "n_select = %d: need 1 <= n_select <= nK = %d", n_select, nK);
  if (nK > 16384) return fail(ctx, ISA_ERR_UNSUPPORTED, "nK = %d key blocks: at most 16384 are built", nK);
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int rows = shape->batch * shape->heads * shape->num_groups;
  ISA_TRY(cuda_status(ctx, launch_top_p_count(mass, rows, nK, top_p, n_select, n_exact_rows, ctx->d_status, st),
                      "isa_select_top_p"));
  return do_select(ctx, shape, mass, n_select, 0, seed, idx, log_w, st, 0, 0, n_exact_rows);
}

size_t isa_cluster_workspace_bytes(const isa_shape* shape, int32_t n_clusters) {
  if (!shape || n_clusters < 1 || n_clusters > kMaxClusters || shape->batch < 1 || shape->heads < 1 ||
      shape->head_dim < 1)
    return 0;
  return cluster_ws(shape, n_clusters);
}

isa_status isa_cluster(isa_context* ctx, const isa_shape* shape, const void* x, int32_t n_clusters, int32_t n_iters,
                       float* centroids, int32_t* labels, int32_t* perm, int32_t* offsets, int32_t* groups,
                       int32_t* n_groups, void* workspace, size_t workspace_bytes, void* stream) {
  ISA_TRY(check_rows_shape(ctx, shape));
  ISA_TRY(check_clusters(ctx, shape, n_clusters));
  if (n_iters < 1 || n_iters > 1000) return fail(ctx, ISA_ERR_INVALID_ARG, "n_iters = %d: need 1..1000", n_iters);
  ISA_TRY(check_ptr(ctx, x, "x", 16));
  ISA_TRY(check_ptr(ctx, centroids, "centroids", 16));
  ISA_TRY(check_ptr(ctx, labels, "labels", 4));
  ISA_TRY(check_ptr(ctx, perm, "perm", 4));
  ISA_TRY(check_ptr(ctx, offsets, "offsets", 4));
  if ((groups == nullptr) != (n_groups == nullptr))
    return fail(ctx, ISA_ERR_INVALID_ARG, "groups and n_groups are given together or not at all");
  if (groups) {
    ISA_TRY(check_ptr(ctx, groups, "groups", 4));
    ISA_TRY(check_ptr(ctx, n_groups, "n_groups", 4));
  }
  ISA_TRY(check_ptr(ctx, workspace, "workspace", 16));
  if (workspace_bytes < cluster_ws(shape, n_clusters))
    return fail(ctx, ISA_ERR_INVALID_ARG, "workspace of %zu bytes, %zu needed", workspace_bytes,
                cluster_ws(shape, n_clusters));
  DeviceGuard g(ctx->device);
  if (!g.ok()) return fail(ctx, ISA_ERR_CUDA, "cannot select device %d", ctx->device);
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  ClusterLaunch l = cluster_launch(shape, n_clusters, x, centroids, workspace);
  l.labels = labels;
  l.perm = perm;
  l.offsets = offsets;
  ISA_TRY(cuda_status(ctx, launch_cluster_init(l, st), "isa_cluster"));
  for (int it = 0; it < n_iters; ++it) {
    const bool last = it == n_iters - 1;
    l.groups = last ? groups : nullptr;
    l.n_groups = last ? n_groups : nullptr;
    ISA_TRY(cuda_status(ctx, launch_cluster_assign(l, ctx->num_sms, ctx->wait_timeout_ns, ctx->d_status, st), "isa_cluster"));
    ISA_TRY(cuda_status(ctx, launch_cluster_sort(l, ctx->d_status, st), "isa_cluster"));
    ISA_TRY(cuda_status(ctx, launch_cluster_update(l, st), "isa_cluster"));
  }
  return ISA_OK;
}

isa_status isa_cluster_assign(isa_context* ctx, const isa_shape* shape, const void* x, const float* centroids,
                              int32_t n_clusters, int32_t* labels, void* workspace, size_t workspace_bytes,
                              void* stream) {
  ISA_TRY(check_rows_shape(ctx, shape));
  ISA_TRY(check_clusters(ctx, shape, n_clusters));
  ISA_TRY(check_ptr(ctx, x, "x", 16));
  ISA_TRY(check_ptr(ctx, centroids, "centroids", 4));
  ISA_TRY(check_ptr(ctx, labels, "labels", 4));
  ISA_TRY(check_ptr(ctx, workspace, "workspace", 16));
  if (workspace_bytes < cluster_ws(shape, n_clusters))
    return fail(ctx, ISA_ERR_INVALID_ARG, "workspace of %zu bytes, %zu needed", workspace_bytes,
                cluster_ws(shape, n_clusters));
  DeviceGuard g(ctx->device);
  if (!g.ok()) return fail(ctx, ISA_ERR_CUDA, "cannot select device %d", ctx->device);
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  ClusterLaunch l = cluster_launch(shape, n_clusters, x, const_cast<float*>(centroids), workspace);
  l.labels = labels;
  ISA_TRY(cuda_status(ctx, launch_cluster_prep(l, st), "isa_cluster_assign"));
  return cuda_status(ctx, launch_cluster_assign(l, ctx->num_sms, ctx->wait_timeout_ns, ctx->d_status, st), "isa_cluster_assign");
}

isa_status isa_cluster_sort(isa_context* ctx, const isa_shape* shape, const int32_t* labels, int32_t n_clusters,
                            int32_t* perm, int32_t* offsets, int32_t* groups, int32_t* n_groups, void* stream) {
  ISA_TRY(check_rows_shape(ctx, shape));
  ISA_TRY(check_clusters(ctx, shape, n_clusters));
  ISA_TRY(check_ptr(ctx, labels, "labels", 4));
  ISA_TRY(check_ptr(ctx, perm, "perm", 4));
  ISA_TRY(check_ptr(ctx, offsets, "offsets", 4));
  if ((groups == nullptr) != (n_groups == nullptr))
    return fail(ctx, ISA_ERR_INVALID_ARG, "groups and n_groups are given together or not at all");
  DeviceGuard g(ctx->device);
  if (!g.ok()) return fail(ctx, ISA_ERR_CUDA, "cannot select device %d", ctx->device);
  ClusterLaunch l{};
  l.BH = shape->batch * shape->heads;
  l.N = shape->seq_len;
  l.D = shape->head_dim;
  l.C = n_clusters;
  l.labels = const_cast<int32_t*>(labels);
  l.perm = perm;
  l.offsets = offsets;
  l.groups = groups;
  l.n_groups = n_groups;
  return cuda_status(ctx, launch_cluster_sort(l, ctx->d_status, static_cast<cudaStream_t>(stream)),
                     "isa_cluster_sort");
}

isa_status isa_cluster_update(isa_context* ctx, const isa_shape* shape, const void* x, const int32_t* perm,
                              const int32_t* offsets, int32_t n_clusters, float* centroids, void* workspace,
                              size_t workspace_bytes, void* stream) {
  ISA_TRY(check_rows_shape(ctx, shape));
  ISA_TRY(check_clusters(ctx, shape, n_clusters));
  ISA_TRY(check_ptr(ctx, x, "x", 16));
  ISA_TRY(check_ptr(ctx, perm, "perm", 4));
  ISA_TRY(check_ptr(ctx, offsets, "offsets", 4));
  ISA_TRY(check_ptr(ctx, centroids, "centroids", 16));
  ISA_TRY(check_ptr(ctx, workspace, "workspace", 16));
  if (workspace_bytes < cluster_ws(shape, n_clusters))
    return fail(ctx, ISA_ERR_INVALID_ARG, "workspace of %zu bytes, %zu needed", workspace_bytes,
                cluster_ws(shape, n_clusters));
  DeviceGuard g(ctx->device);
  if (!g.ok()) return fail(ctx, ISA_ERR_CUDA, "cannot select device %d", ctx->device);
  ClusterLaunch l = cluster_launch(shape, n_clusters, x, centroids, workspace);
  l.perm = const_cast<int32_t*>(perm);
  l.offsets = const_cast<int32_t*>(offsets);
  return cuda_status(ctx, launch_cluster_update(l, static_cast<cudaStream_t>(stream)), "isa_cluster_update");
}

isa_status isa_permute_rows(isa_context* ctx, const isa_shape* shape, const void* x, const int32_t* perm,
                            int32_t inverse, void* out, void* stream) {
  ISA_TRY(check_rows_shape(ctx, shape));
  ISA_TRY(check_ptr(ctx, x, "x", 16));
  ISA_TRY(check_ptr(ctx, perm, "perm", 4));
  ISA_TRY(check_ptr(ctx, out, "out", 16));
  if (x == out) return fail(ctx, ISA_ERR_INVALID_ARG, "x and out must not be the same buffer");
  DeviceGuard g(ctx->device);
  if (!g.ok()) return fail(ctx, ISA_ERR_CUDA, "cannot select device %d", ctx->device);
  return cuda_status(ctx,
                     launch_permute_rows(x, perm, shape->batch * shape->heads, shape->seq_len, shape->head_dim,
                                         inverse != 0, out, ctx->d_status, ctx->num_sms,
                                         static_cast<cudaStream_t>(stream)),
                     "isa_permute_rows");
}

size_t isa_attention_workspace_bytes(const isa_shape* s) { return s ? attn_ws_bytes(s) : 0; }

isa_status isa_attention(isa_context* ctx, const isa_shape* shape, const void* q, const void* k, const void* v,
                         const int32_t* idx, const float* log_w, int32_t n_sel, void* out, float* lse,
                         void* workspace, size_t workspace_bytes, void* stream) {
  ISA_TRY(check_shape(ctx, shape));
  DeviceGuard g(ctx->device);
  if (!g.ok()) return fail(ctx, ISA_ERR_CUDA, "cannot select device %d", ctx->device);
  return do_attention(ctx, shape, q, k, v, idx, log_w, n_sel, out, lse, workspace, workspace_bytes, false,
                      static_cast<cudaStream_t>(stream));
}

isa_status isa_dense_attention(isa_context* ctx, const isa_shape* shape, const void* q, const void* k,
                               const void* v, void* out, float* lse, void* stream) {
  ISA_TRY(check_shape(ctx, shape));
  DeviceGuard g(ctx->device);
  if (!g.ok()) return fail(ctx, ISA_ERR_CUDA, "cannot select device %d", ctx->device);
  return do_attention(ctx, shape, q, k, v, nullptr, nullptr, 0, out, lse, nullptr, 0, true,
                      static_cast<cudaStream_t>(stream));
}

size_t isa_tail_merge_workspace_bytes(const isa_shape* s, int32_t n_sel) {
  if (!s || s->batch < 1 || s->heads < 1 || s->num_groups < 1 || s->seq_len < 1 || s->k_block < 1 || n_sel < 1)
    return 0;
  return merge_carve(s->batch * s->heads, s->seq_len, s->num_groups, n_sel, nblocks(s)).total;
}

isa_status isa_tail_merge(isa_context* ctx, const isa_shape* shape, const int32_t* idx, const float* log_w,
                          int32_t n_sel, void* schedule, size_t schedule_bytes, void* stream) {
  ISA_TRY(check_shape(ctx, shape));
  if (!shape->q_offsets) return fail(ctx, ISA_ERR_INVALID_ARG, "tail merging needs q_offsets (the permuted layout)");
  ISA_TRY(check_ptr(ctx, idx, "idx", 4));
  ISA_TRY(check_ptr(ctx, log_w, "log_w", 4));
  if (n_sel < 1) return fail(ctx, ISA_ERR_INVALID_ARG, "n_sel must be >= 1");
  const size_t need = isa_tail_merge_workspace_bytes(shape, n_sel);
  if (!schedule || schedule_bytes < need)
    return fail(ctx, ISA_ERR_INVALID_ARG, "schedule %zu bytes < %zu needed", schedule_bytes, need);
  if (!aligned(schedule, 256)) return fail(ctx, ISA_ERR_INVALID_ARG, "schedule not 256-byte aligned");
  DeviceGuard g(ctx->device);
  if (!g.ok()) return fail(ctx, ISA_ERR_CUDA, "cannot select device %d", ctx->device);
  const int BH = shape->batch * shape->heads;
  const MergeCarve c = merge_carve(BH, shape->seq_len, shape->num_groups, n_sel, nblocks(shape));
  char* w = static_cast<char*>(schedule);
  MergeLaunch m{};
  m.BH = BH;
  m.N = shape->seq_len;
  m.G = shape->num_groups;
  m.S = n_sel;
  m.Bk = shape->k_block;
  m.nK = nblocks(shape);
  m.W = (m.nK + 31) / 32;
  m.q_offsets = shape->q_offsets;
  m.idx = idx;
  m.log_w = log_w;
  m.bins = reinterpret_cast<MergeBin*>(w + c.bins);
  m.counts = reinterpret_cast<int32_t*>(w + c.counts);
  m.order = reinterpret_cast<int32_t*>(w + c.order);
  m.state = reinterpret_cast<uint32_t*>(w + c.state);
  m.prefix = reinterpret_cast<int32_t*>(w + c.prefix);
  m.unions = reinterpret_cast<int32_t*>(w + c.unions);
  m.tables = reinterpret_cast<float*>(w + c.tables);
  m.items = reinterpret_cast<WorkItem*>(w + c.items);
  m.item_count = reinterpret_cast<int32_t*>(w + c.item_count);
  m.status = ctx->d_status;
  {
    // the attention's grid for these items (isa_attention_merged launches the same)
    const long long pairs = (static_cast<long long>(BH) * (m.G + m.N / 128) + 1) / 2;
    m.grid = static_cast<int>(pairs < ctx->num_sms ? pairs : ctx->num_sms);
  }
  return cuda_status(ctx, launch_tail_merge(m, static_cast<cudaStream_t>(stream)), "isa_tail_merge");
}

isa_status isa_attention_merged(isa_context* ctx, const isa_shape* shape, const void* q, const void* k, const void* v,
                                const int32_t* idx, const float* log_w, int32_t n_sel, const void* schedule,
                                size_t schedule_bytes, void* out, float* lse, void* stream) {
  ISA_TRY(check_shape(ctx, shape));
  if (!shape->q_offsets) return fail(ctx, ISA_ERR_INVALID_ARG, "merged attention needs q_offsets");
  ISA_TRY(check_ptr(ctx, q, "q", 16));
  ISA_TRY(check_ptr(ctx, k, "k", 16));
  ISA_TRY(check_ptr(ctx, v, "v", 16));
  ISA_TRY(check_ptr(ctx, out, "out", 16));
  ISA_TRY(check_ptr(ctx, idx, "idx", 4));
  ISA_TRY(check_ptr(ctx, log_w, "log_w", 4));
  if (lse && !aligned(lse, 4)) return fail(ctx, ISA_ERR_INVALID_ARG, "lse not 4-byte aligned");
  if (n_sel < 1) return fail(ctx, ISA_ERR_INVALID_ARG, "n_sel must be >= 1");
  const size_t need = isa_tail_merge_workspace_bytes(shape, n_sel);
  if (!schedule || schedule_bytes < need)
    return fail(ctx, ISA_ERR_INVALID_ARG, "schedule %zu bytes < %zu needed", schedule_bytes, need);
  if (!aligned(schedule, 256)) return fail(ctx, ISA_ERR_INVALID_ARG, "schedule not 256-byte aligned");
  DeviceGuard g(ctx->device);
  if (!g.ok()) return fail(ctx, ISA_ERR_CUDA, "cannot select device %d", ctx->device);
  const MergeCarve c =
      merge_carve(shape->batch * shape->heads, shape->seq_len, shape->num_groups, n_sel, nblocks(shape));
  const char* w = static_cast<const char*>(schedule);
  AttnLaunch l{};
  l.B = shape->batch;
  l.H = shape->heads;
  l.N = shape->seq_len;
  l.D = shape->head_dim;
  l.G = shape->num_groups;
  l.S = n_sel;
  l.Bk = shape->k_block;
  l.q_block = shape->q_block;
  l.mode = kAttnMerged;
  l.q_offsets = shape->q_offsets;
  l.idx = idx;
  l.log_w = log_w;
  l.out = out;
  l.lse = lse;
  l.scale = shape->scale;
  l.status = ctx->d_status;
  l.num_sms = ctx->num_sms;
  l.wait_timeout_ns = ctx->wait_timeout_ns;
  l.stall = ctx->stall_attention;
  l.items = reinterpret_cast<const WorkItem*>(w + c.items);
  l.item_count = reinterpret_cast<const int32_t*>(w + c.item_count);
  l.bins = reinterpret_cast<const MergeBin*>(w + c.bins);
  l.unions = reinterpret_cast<const int32_t*>(w + c.unions);
  l.tables = reinterpret_cast<const float*>(w + c.tables);
  return cuda_status(ctx, launch_attention_merged(l, q, k, v, static_cast<cudaStream_t>(stream)),
                     "isa_attention_merged");
}

size_t isa_plan_workspace_bytes(const isa_shape* s, const isa_params* p) {
  if (!s || !p || p->n_clusters < 1 || s->heads < 1 || s->num_groups < 1 || s->k_block < 1) return 0;
  return plan_bytes(s, p);
}

isa_status isa_plan(isa_context* ctx, const isa_shape* shape, const isa_params* params, const void* q, const void* k,
                    int32_t* idx, float* log_w, void* workspace, size_t workspace_bytes, void* stream) {
  ISA_TRY(check_shape(ctx, shape));
  if (!params) return fail(ctx, ISA_ERR_INVALID_ARG, "params is NULL");
  if (params->n_clusters < 1 || params->n_clusters > 16) return fail(ctx, ISA_ERR_INVALID_ARG, "n_clusters must be 1..16");
  ISA_TRY(check_ptr(ctx, q, "q", 16));
  ISA_TRY(check_ptr(ctx, k, "k", 16));
  ISA_TRY(check_ptr(ctx, idx, "idx", 4));
  ISA_TRY(check_ptr(ctx, log_w, "log_w", 4));
  const size_t need = plan_bytes(shape, params);
  if (!workspace || workspace_bytes < need)
    return fail(ctx, ISA_ERR_INVALID_ARG, "plan workspace %zu bytes < %zu needed", workspace_bytes, need);
  if (!aligned(workspace, 256)) return fail(ctx, ISA_ERR_INVALID_ARG, "workspace not 256-byte aligned");
  DeviceGuard g(ctx->device);
  if (!g.ok()) return fail(ctx, ISA_ERR_CUDA, "cannot select device %d", ctx->device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int H = shape->heads, hc = plan_chunk_heads(shape);
  const size_t G = static_cast<size_t>(shape->num_groups), S = static_cast<size_t>(params->n_exact) + params->n_sample;
  const size_t head_elems = static_cast<size_t>(shape->seq_len) * shape->head_dim;
  const size_t score_ws = round_up(
      score_workspace_bytes(1, hc, shape->seq_len, shape->head_dim, shape->num_groups, shape->k_block, params->n_clusters));
  char* w = static_cast<char*>(workspace);
  float* mass = reinterpret_cast<float*>(w + score_ws);
  // Chunks of heads: score the chunk into the chunk-sized mass buffer, then
  // select from it while it is still in L2; the selector drops every line it
  // has read, so the mass is not written back to HBM.  Heads are independent
  // and the uniforms are keyed by the global head and batch index, so the
  // plan is the one isa_select(isa_score(.)) gives on the whole layer.
  for (int b = 0; b < shape->batch; ++b) {
    for (int h0 = 0; h0 < H; h0 += hc) {
      const int nh = H - h0 < hc ? H - h0 : hc;
      isa_shape sub = *shape;
      sub.batch = 1;
      sub.heads = nh;
      const size_t bh0 = static_cast<size_t>(b) * H + h0;
      const char* qc = static_cast<const char*>(q) + bh0 * head_elems * 2;
      const char* kc = static_cast<const char*>(k) + bh0 * head_elems * 2;
      ISA_TRY(do_score(ctx, &sub, qc, kc, params->n_clusters, params->n_iters, mass, nullptr, nullptr, w, score_ws,
                       st));
      ISA_TRY(do_select(ctx, &sub, mass, params->n_exact, params->n_sample, params->seed, idx + bh0 * G * S,
                        log_w + bh0 * G * S, st, h0, b, nullptr, true));
    }
  }
  return ISA_OK;
}

size_t isa_pipeline_workspace_bytes(const isa_shape* s, const isa_params* p) {
  if (!s || !p || p->n_clusters < 1) return 0;
  return pipeline_bytes(s, p);
}

isa_status isa_pipeline(isa_context* ctx, const isa_shape* shape, const isa_params* params, const void* q,
                        const void* k, const void* v, void* out, float* lse, int32_t* plan_idx, float* plan_log_w,
                        void* workspace, size_t workspace_bytes, void* stream) {
  ISA_TRY(check_shape(ctx, shape));
  DeviceGuard g(ctx->device);
  if (!g.ok()) return fail(ctx, ISA_ERR_CUDA, "cannot select device %d", ctx->device);
  return do_pipeline(ctx, shape, params, q, k, v, out, lse, plan_idx, plan_log_w, workspace, workspace_bytes,
                     static_cast<cudaStream_t>(stream));
}

size_t isa_pipeline_host_workspace_bytes(const isa_shape* s, const isa_params* p) {
  if (!s || !p || p->n_clusters < 1) return 0;
  const size_t t = round_up(static_cast<size_t>(s->batch) * s->heads * s->seq_len * s->head_dim * 2);
  return 4 * t + pipeline_bytes(s, p);
}

isa_status isa_pipeline_host(isa_context* ctx, const isa_shape* shape, const isa_params* params, const void* q_host,
                             const void* k_host, const void* v_host, void* out_host, void* workspace,
                             size_t workspace_bytes, void* stream) {
  ISA_TRY(check_shape(ctx, shape));
  if (!params) return fail(ctx, ISA_ERR_INVALID_ARG, "params is NULL");
  if (!q_host || !k_host || !v_host || !out_host) return fail(ctx, ISA_ERR_INVALID_ARG, "host buffer is NULL");
  const size_t need = isa_pipeline_host_workspace_bytes(shape, params);
  if (!workspace || workspace_bytes < need)
    return fail(ctx, ISA_ERR_INVALID_ARG, "host-pipeline arena %zu bytes < %zu needed", workspace_bytes, need);
  if (!aligned(workspace, 256)) return fail(ctx, ISA_ERR_INVALID_ARG, "workspace not 256-byte aligned");
  DeviceGuard g(ctx->device);
  if (!g.ok()) return fail(ctx, ISA_ERR_CUDA, "cannot select device %d", ctx->device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t bytes = static_cast<size_t>(shape->batch) * shape->heads * shape->seq_len * shape->head_dim * 2;
  const size_t t = round_up(bytes);
  char* w = static_cast<char*>(workspace);
  char *dq = w, *dk = w + t, *dv = w + 2 * t, *dout = w + 3 * t;
  // The layer runs in chunks of heads so that copies overlap the compute:
  // chunk i's inputs go up on one copy stream while chunk i-1 computes on
  // `stream` and chunk i-2's output comes down on another.  Heads are
  // independent, and the selector keys its uniform by the global head and
  // batch index, so the result is the one isa_pipeline gives on the whole
  // layer.
  if (!ctx->copy_in && cudaStreamCreateWithFlags(&ctx->copy_in, cudaStreamNonBlocking) != cudaSuccess)
    return fail(ctx, ISA_ERR_CUDA, "isa_pipeline_host: cannot create a copy stream");
  if (!ctx->copy_out && cudaStreamCreateWithFlags(&ctx->copy_out, cudaStreamNonBlocking) != cudaSuccess)
    return fail(ctx, ISA_ERR_CUDA, "isa_pipeline_host: cannot create a copy stream");
  const int H = shape->heads;
  const int hc = (H + 15) / 16;  // heads per chunk: up to 16 chunks per batch entry
  const size_t head_bytes = static_cast<size_t>(shape->seq_len) * shape->head_dim * 2;
  std::vector<cudaEvent_t> evs;
  auto new_event = [&](cudaEvent_t* ev) -> bool {
    if (cudaEventCreateWithFlags(ev, cudaEventDisableTiming) != cudaSuccess) return false;
    evs.push_back(*ev);
    return true;
  };
  auto release = [&]() {
    for (cudaEvent_t ev : evs) cudaEventDestroy(ev);  // pending records complete first
  };
  isa_status result = ISA_OK;
  cudaError_t e = cudaSuccess;
  cudaEvent_t start;
  // nothing may overwrite the arena before earlier work on `stream` is done
  if (!new_event(&start) || (e = cudaEventRecord(start, st)) != cudaSuccess ||
      (e = cudaStreamWaitEvent(ctx->copy_in, start, 0)) != cudaSuccess ||
      (e = cudaStreamWaitEvent(ctx->copy_out, start, 0)) != cudaSuccess) {
    release();
    return fail(ctx, ISA_ERR_CUDA, "isa_pipeline_host: event setup failed");
  }
  for (int b = 0; b < shape->batch && result == ISA_OK; ++b) {
    for (int h0 = 0; h0 < H && result == ISA_OK; h0 += hc) {
      const int nh = H - h0 < hc ? H - h0 : hc;
      const size_t off = (static_cast<size_t>(b) * H + h0) * head_bytes, len = static_cast<size_t>(nh) * head_bytes;
      cudaEvent_t in_done, comp_done;
      if (!new_event(&in_done) || !new_event(&comp_done)) {
        result = fail(ctx, ISA_ERR_CUDA, "isa_pipeline_host: cannot create an event");
        break;
      }
      e = cudaMemcpyAsync(dq + off, static_cast<const char*>(q_host) + off, len, cudaMemcpyHostToDevice, ctx->copy_in);
      if (e == cudaSuccess)
        e = cudaMemcpyAsync(dk + off, static_cast<const char*>(k_host) + off, len, cudaMemcpyHostToDevice,
                            ctx->copy_in);
      if (e == cudaSuccess)
        e = cudaMemcpyAsync(dv + off, static_cast<const char*>(v_host) + off, len, cudaMemcpyHostToDevice,
                            ctx->copy_in);
      if (e == cudaSuccess) e = cudaEventRecord(in_done, ctx->copy_in);
      if (e == cudaSuccess) e = cudaStreamWaitEvent(st, in_done, 0);
      if (e != cudaSuccess) {
        result = fail(ctx, ISA_ERR_CUDA, "isa_pipeline_host copy in: %s", cudaGetErrorString(e));
        break;
      }
      isa_shape sub = *shape;
      sub.batch = 1;
      sub.heads = nh;
      result = do_pipeline(ctx, &sub, params, dq + off, dk + off, dv + off, dout + off, nullptr, nullptr, nullptr,
                           w + 4 * t, need - 4 * t, st, h0, b);
      if (result != ISA_OK) break;
      e = cudaEventRecord(comp_done, st);
      if (e == cudaSuccess) e = cudaStreamWaitEvent(ctx->copy_out, comp_done, 0);
      if (e == cudaSuccess)
        e = cudaMemcpyAsync(static_cast<char*>(out_host) + off, dout + off, len, cudaMemcpyDeviceToHost,
                            ctx->copy_out);
      if (e != cudaSuccess) result = fail(ctx, ISA_ERR_CUDA, "isa_pipeline_host copy out: %s", cudaGetErrorString(e));
    }
  }
  // `stream` completes only after the last output copy (and, on an error, after
  // whatever was enqueued on the copy streams)
  cudaEvent_t fin_in, fin_out;
  if (new_event(&fin_in) && new_event(&fin_out)) {
    cudaEventRecord(fin_in, ctx->copy_in);
    cudaEventRecord(fin_out, ctx->copy_out);
    cudaStreamWaitEvent(st, fin_in, 0);
    cudaStreamWaitEvent(st, fin_out, 0);
  } else if (result == ISA_OK) {
    result = fail(ctx, ISA_ERR_CUDA, "isa_pipeline_host: cannot create an event");
  }
  release();
  return result;
}

}  // extern "C"

namespace isa_impl {

cudaError_t ensure_smem_attr(const void* func, int bytes) {
  struct Entry {
    const void* func;
    int device, bytes;
  };
  static std::mutex mu;
  static std::vector<Entry> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  for (const Entry& x : done)
    if (x.func == func && x.device == dev && x.bytes >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  for (Entry& x : done)
    if (x.func == func && x.device == dev) {
      x.bytes = bytes;
      return cudaSuccess;
    }
  done.push_back({func, dev, bytes});
  return cudaSuccess;
}

}  // namespace isa_impl

// ---------------------------------------------------------------------------
// isa_attention_noalloc: isa_attention for callers that cannot allocate.
//
// Some callers cannot hand this library any device memory of their own: a
// framework custom-op or plugin interface that passes a kernel only its
// inputs and outputs, or latency-critical code that must not call cudaMalloc
// (which may synchronise the device) and has no workspace to lend.  For
// them the tile-list scratch of the attention kernel (needed for variable
// query clusters and for uniform groups of more than 128 rows) lives in the
// file-scope array below instead of a caller workspace.
//
// The array is a module global: every GPU that loads this library holds its
// kNoAllocScratchBytes until the process exits.  In host code its name is only
// a host-side stand-in, so the device address is looked up with
// cudaGetSymbolAddress the first time the entry point runs on a device (with
// that device current) and cached per device.  Make that first call on each
// device before any stream capture.  A device reset may move the array and
// leave the cached address stale, so the entry point is not for use after one.  Every call shares the one array and it
// keeps the last call's contents; the tile-list kernel rewrites every entry it
// uses (and the count) on each call, so nothing needs clearing.  Calls whose
// kernels overlap on the GPU (different streams, no ordering between them)
// race on the array.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(1) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[64] = {nullptr};

// Device address of the scratch array on `device` (which must be current).
cudaError_t noalloc_scratch(int device, void** out) {
  if (device < 0 || device >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (!g_noalloc_ptr[device]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_noalloc_ptr[device] = p;
  }
  *out = g_noalloc_ptr[device];
  return cudaSuccess;
}

}  // namespace

extern "C" isa_status isa_attention_noalloc(isa_context* ctx, const isa_shape* shape, const void* q, const void* k,
                                            const void* v, const int32_t* idx, const float* log_w, int32_t n_sel,
                                            void* out, float* lse, void* stream) {
  ISA_TRY(check_shape(ctx, shape));
  const size_t need = attn_ws_bytes(shape);
  if (need > kNoAllocScratchBytes)
    return fail(ctx, ISA_ERR_INVALID_ARG,
                "isa_attention_noalloc: the tile list needs %zu bytes, more than its built-in %zu-byte scratch "
                "(num_groups + seq_len/128 must stay below %zu); use isa_attention with a workspace",
                need, kNoAllocScratchBytes, kNoAllocScratchBytes / 16 - 1);
  DeviceGuard g(ctx->device);
  if (!g.ok()) return fail(ctx, ISA_ERR_CUDA, "cannot select device %d", ctx->device);
  void* scratch = nullptr;
  if (need) {
    const cudaError_t e = noalloc_scratch(ctx->device, &scratch);
    if (e != cudaSuccess)
      return fail(ctx, ISA_ERR_CUDA, "isa_attention_noalloc: cudaGetSymbolAddress: %s", cudaGetErrorString(e));
  }
  return do_attention(ctx, shape, q, k, v, idx, log_w, n_sel, out, lse, scratch, need ? kNoAllocScratchBytes : 0,
                      false, static_cast<cudaStream_t>(stream));
}
