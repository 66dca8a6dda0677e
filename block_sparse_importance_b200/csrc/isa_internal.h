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

// ---------------------------------------------------------- tail merging
// One tile of cluster tails (1..4 members) of one (batch, head), and the
// attention's work items, as isa_tail_merge lays them out in its workspace.
struct MergeBin {
  int32_t n;     // members
  int32_t rows;  // rows taken by the members' 32-row slots
  int32_t ulen;  // blocks in the union of the members' plans
  int32_t uoff;  // first union entry in the head's union pool (tiles of 2+ members)
  int32_t toff;  // first entry of the [n][ulen] log-weight table in the head's pool
  int32_t pad[3];
  int32_t g[4];     // member clusters (-1 past the last)
  int32_t slot[4];  // first tile row of each member
};
struct WorkItem {
  int32_t bh;
  int32_t g;  // >= 0: rows [row0, row0 + nrows) of cluster g on its plan row; < 0: tile -1 - g of head bh
  int32_t row0, nrows;
};
struct MergeLaunch {
  int BH, N, G, S, Bk, nK, W;  // W = 32-bit words of an nK-bit mask
  const int32_t* q_offsets;    // device [G+1]
  const int32_t* idx;          // [BH, G, S]
  const float* log_w;          // [BH, G, S]
  MergeBin* bins;              // [BH][G]
  int32_t* counts;             // [BH][2]: tiles of tails, merged tiles among them
  int32_t* order;              // [BH][G] scratch: the tails in schedule order
  uint32_t* state;             // [BH][merge_state_words] scratch, when not in shared memory
  int32_t* prefix;             // [BH][8][W] scratch: per-warp word prefixes
  int32_t* unions;             // [BH][G S]: union lists, ascending
  float* tables;               // [BH][4 G S]: log-weights per member and union position
  WorkItem* items;             // [BH (N / 128 + G)]
  int32_t* item_count;
  int state_in_smem;
  int grid;  // CTAs of the attention that runs the items (merged tiles are spread over them)
  int* status;
};
// the greedy's state per (b, h), in 32-bit words: rows, members and union
// size of every tile, two plan masks and the tiles' union masks
__host__ __device__ inline size_t merge_state_words(int G, int W) {
  return 3 * static_cast<size_t>(G) + 2 * static_cast<size_t>(W) + static_cast<size_t>(G) * W;
}
// byte offsets of the parts of the workspace
struct MergeCarve {
  size_t bins, counts, order, state, prefix, unions, tables, items, item_count, total;
};
MergeCarve merge_carve(int BH, int N, int G, int S, int nK);
constexpr size_t kMergeSmemState = 160 * 1024;  // the greedy's state up to this size stays in shared memory
int launch_tail_merge(const MergeLaunch& m, cudaStream_t stream);

// ------------------------------------------------------------- attention
enum AttnMode : int {
  kAttnGroups = 0,  // uniform query groups of <= 128 rows: one tile per group
  kAttnList = 1,    // tile list built on the device (clusters or groups > 128 rows)
  kAttnDense = 2,   // all keys, no plan
  kAttnMerged = 3   // work items of isa_tail_merge: cluster tiles and merged tail tiles
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
  // kAttnMerged: the schedule of isa_tail_merge
  const WorkItem* items;
  const int32_t* item_count;
  const MergeBin* bins;   // [B H][G]
  const int32_t* unions;  // [B H][G S]
  const float* tables;    // [B H][4 G S]
};

size_t attn_list_workspace_bytes(int N, int G);
// kAttnMerged (attn_merged.cu): the schedule of isa_tail_merge.
int launch_attention_merged(const AttnLaunch& a, const void* q, const void* k, const void* v, cudaStream_t stream);
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
  uint32_t* kb_next;  // scratch: the next key block to take (key means beside the k-means)
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
