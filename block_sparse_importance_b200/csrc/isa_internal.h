// Internal launch interface between the C-ABI layer (isa_api.cu) and the
// kernels.  Not part of the public ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace isa_impl {

// Device status codes (same values as isa_status).
enum : int { kStatusOk = 0, kStatusTimeout = 4, kStatusDeviceCheck = 5 };

// Per-wait time limit of every bounded pipeline wait in the kernels.
constexpr uint64_t kWaitTimeoutNs = 2000000000ull;

// Opts `func` into `bytes` of dynamic shared memory on the current device.
// The attribute belongs to the function in the current device's context, so a
// process that drives several GPUs needs it once per (function, device); the
// record of what has been set is kept under a mutex.
cudaError_t ensure_smem_attr(const void* func, int bytes);

// ------------------------------------------------------------- attention
enum AttnMode : int {
  kAttnGroups = 0,  // uniform query groups of <= 128 rows: one tile per group
  kAttnList = 1,    // tile list built on the device (clusters or groups > 128 rows)
  kAttnDense = 2    // all keys, no plan
};

struct AttnLaunch {
  int B, H, N, D, G, S, Bk, q_block;
  int mode;
  const int32_t* q_offsets;  // kAttnList: device [G+1] (NULL: uniform q_block groups)
  const int32_t* idx;
  const float* log_w;
  void* out;
  float* lse;
  void* workspace;           // kAttnList: tile list + count
  float scale;
  int* status;
  int num_sms;
  uint64_t wait_timeout_ns;  // per-wait limit of the bounded pipeline waits
  int stall;                 // test hook: the MMA warp waits on a barrier nothing arrives at
};

size_t attn_list_workspace_bytes(int N, int G);
// Builds tensor maps for q/k/v and launches.  Returns a cudaError_t value or
// -1 if a tensor map could not be encoded.
int launch_attention(const AttnLaunch& a, const void* q, const void* k, const void* v,
                     cudaStream_t stream);

// -------------------------------------------------------------- selector
struct SelectLaunch {
  int B, H, G, nK, n_exact, n_sample;
  int h_base, b_base;  // head and batch index of the launch's first row in the whole tensor
  uint64_t seed;
  const float* mass;
  int32_t* idx;
  float* log_w;
  // per-row exact-set sizes (top-p rule), or NULL for the fixed n_exact; with
  // it, n_exact + n_sample is the plan size and row r uses ne_rows[r] exact
  const int32_t* ne_rows;
  int* status;
  int num_sms;
  // the mass is scratch: once a row has been read, its whole 128-byte lines
  // are dropped from L2 without being written back (discard.global.L2)
  int discard_mass;
};
int launch_select(const SelectLaunch& s, cudaStream_t stream);
// Exact-set sizes under the top-p rule, one per plan row, into ne_rows.
int launch_top_p_count(const float* mass, int rows, int nK, double top_p, int S, int32_t* ne_rows, int* status,
                       cudaStream_t stream);

// ---------------------------------------------------------------- scorer
struct ScoreLaunch {
  int B, H, N, D, G, Bk, q_block, C, iters;
  const int32_t* q_offsets;  // device or NULL
  float scale;
  const void* q;
  const void* k;
  float* mass;
  float* centroids;   // [B,H,G,C,D]
  int32_t* counts;    // [B,H,G,C]
  uint16_t* kbar_hi;  // [B,H,nK,D] bf16 scratch: key-block means, high part
  uint16_t* kbar_lo;  // [B,H,nK,D] bf16 scratch: key-block means, low part
  int* status;
  int num_sms;
};
size_t score_workspace_bytes(int B, int H, int N, int D, int G, int Bk, int C);
int launch_score(const ScoreLaunch& s, cudaStream_t stream);

// ------------------------------------------------------ token clustering
// k-means over the whole sequence of every (batch, head) and the stable
// counting sort of its labels (the permuted layout).  The centroids' bf16
// hi / lo split and squared norms live in caller scratch, Cpad = C rounded
// up to 128 rows (padding rows: zero, norm +inf).
struct ClusterLaunch {
  int BH, N, D, C, Cpad;
  const void* x;         // [BH, N, D] bf16
  float* mu;             // [BH, C, D]
  uint16_t* mu_hi;       // [BH, Cpad, D]
  uint16_t* mu_lo;       // [BH, Cpad, D]
  float* mu_nsq;         // [BH, Cpad]
  int32_t* labels;       // [BH, N]
  int32_t* perm;         // [BH, N]
  int32_t* offsets;      // [BH, C + 1]
  int32_t* groups;       // [BH, C + 1] or NULL
  int32_t* n_groups;     // [BH] or NULL
};
inline int cluster_cpad(int C) { return (C + 127) / 128 * 128; }
int launch_cluster_init(const ClusterLaunch& l, cudaStream_t stream);     // mu = rows floor(c N / C), then prep
int launch_cluster_prep(const ClusterLaunch& l, cudaStream_t stream);     // hi / lo / norms of mu
int launch_cluster_assign(const ClusterLaunch& l, int num_sms, uint64_t timeout_ns, int* status,
                          cudaStream_t stream);  // labels from hi / lo / norms (tcgen05)
int launch_cluster_sort(const ClusterLaunch& l, int* status, cudaStream_t stream);  // perm, offsets (groups)
int launch_cluster_update(const ClusterLaunch& l, cudaStream_t stream);   // mu (and prep) from perm, offsets
int launch_permute_rows(const void* x, const int32_t* perm, int BH, int N, int D, bool inverse, void* out, int* status,
                        int num_sms, cudaStream_t stream);

}  // namespace isa_impl
