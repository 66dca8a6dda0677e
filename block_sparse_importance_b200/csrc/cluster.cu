// Token clustering for the permuted layout of permuted block-sparse attention.
//
// "InstaGen: Group-Shared Importance Sampling for Fast Video Generation"
// (abstract): permuted block-sparse attention computes blocks of a
// semantically permuted attention matrix, and InstaGen is parameterised by
// the SVG2 method, whose semantic-aware permutation clusters the tokens of
// the whole sequence and reorders them cluster by cluster; "AB-Attention"
// contrasts its own in-block clustering with that sequence-wide clustering
// and token permutation.  Per (batch, head), Lloyd's k-means over all N rows
// with C clusters, centroids initialised at rows floor(c N / C); each round
//   assign  argmin_c ||x - mu_c||^2 = argmin_c (|mu_c|^2 - 2 x.mu_c), ties to
//           the lower c; the dot products run on the tensor cores (tcgen05,
//           fp32 accumulators in TMEM) with x exact in bf16 and mu split into
//           bf16 hi + lo parts (relative error at most 2^-18), two products per k-step
//           (a distance is then within 2^-18 + about 2 d 2^-24 of ||x||^2 + ||mu||^2
//           of the exact one, below 2e-5 of it at d = 128);
//   sort    a stable counting sort of the labels: perm lists the rows in
//           (label, row) order, offsets[c] .. offsets[c + 1] are cluster c's;
//   update  mu_c = the fp32 mean of cluster c's rows taken in permutation
//           order (an empty cluster keeps its centroid).
// A query cluster is then one query group of the attention path, and the
// reordered keys form its key blocks; permute_rows_kernel applies a
// permutation (gather) or its inverse (scatter) to rows of d values.

#include <cuda_bf16.h>

#include <cstdint>

#include "isa_internal.h"
#include "mma_sync.cuh"
#include "ptx.cuh"
#include "tmap.h"

namespace isa_impl {
namespace {

__device__ __forceinline__ float bf16f(uint16_t h) { return __uint_as_float(static_cast<uint32_t>(h) << 16); }

constexpr int kPrepWarps = 8;

// mu_c = row floor(c N / C) of the head, as fp32.  One warp per centroid.
template <int D>
__global__ void __launch_bounds__(kPrepWarps * 32) cluster_init_kernel(ClusterLaunch l) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x * kPrepWarps + warp;
  const int64_t bh = blockIdx.y;
  if (c >= l.C) return;
  constexpr int PER = D / 32;
  const int64_t r = (static_cast<int64_t>(c) * l.N) / l.C;
  const uint16_t* src = static_cast<const uint16_t*>(l.x) + (bh * l.N + r) * D + lane * PER;
  float* dst = l.mu + (bh * l.C + c) * D + lane * PER;
#pragma unroll
  for (int i = 0; i < PER; ++i) dst[i] = bf16f(src[i]);
}

// The assignment's operands of centroid c: hi = bf16(mu), lo = bf16(mu - hi),
// nsq = |mu|^2 (fp32); padding rows c >= C get zeros and nsq = +inf.
template <int D>
__device__ __forceinline__ void write_prep(const ClusterLaunch& l, int64_t bh, int c, const float (&v)[D / 32],
                                           bool live) {
  using namespace isa_dev;
  constexpr int PER = D / 32;
  const int lane = threadIdx.x & 31;
  float s = 0.0f;
  const int64_t o = (bh * l.Cpad + c) * D + lane * PER;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const uint16_t hi = live ? bf16_bits_rn(v[i]) : 0;
    const uint16_t lo = live ? bf16_bits_rn(v[i] - bf16_bits_to_f(hi)) : 0;
    l.mu_hi[o + i] = hi;
    l.mu_lo[o + i] = lo;
    s = fmaf(v[i], v[i], s);
  }
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) s += __shfl_xor_sync(0xffffffffu, s, m);
  if (lane == 0) l.mu_nsq[bh * l.Cpad + c] = live ? s : INFINITY;
}

template <int D>
__global__ void __launch_bounds__(kPrepWarps * 32) cluster_prep_kernel(ClusterLaunch l) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x * kPrepWarps + warp;
  const int64_t bh = blockIdx.y;
  if (c >= l.Cpad) return;
  constexpr int PER = D / 32;
  float v[PER];
  const bool live = c < l.C;
#pragma unroll
  for (int i = 0; i < PER; ++i) v[i] = live ? l.mu[(bh * l.C + c) * D + lane * PER + i] : 0.0f;
  write_prep<D>(l, bh, c, v, live);
}

// Nearest centroid on the tensor cores (tcgen05), a persistent CTA per SM
// walking 128-row tiles of the heads.  Per tile, the centroids come in chunks
// of 128; for each chunk the MMA warp computes S = X hi^T + X lo^T (M = 128
// rows, N = 128 centroids, K = d; two products per k-step) into one of two
// TMEM accumulators, and each epilogue thread (one per row = TMEM lane)
// updates its running argmin of nsq_c - 2 S_c.  Candidates arrive in
// ascending c and a strict compare keeps the first minimum, so ties go to
// the lower c with no cross-lane step.
//   warps 0-3  epilogue (argmin, labels);
//   warp 4     TMA producer: the X tile (two buffers) and the centroid hi / lo
//              chunks (two stages);
//   warp 5     MMA issue (one elected lane of a converged warp).
// Every wait is bounded (global timer + CTA abort flag): on a timeout the CTA
// drains its copies and products, frees TMEM and records ISA_ERR_TIMEOUT.
constexpr int kAsgThreads = 192;
constexpr int kAsgRows = 128;
constexpr int kAsgChunk = 128;  // centroids per stage (the MMA's N)

template <int D>
struct AsgLayout {
  static constexpr uint32_t kTile = 128 * D * 2;  // 128 rows x D bf16, 64-column boxes, 128-byte swizzle
  static constexpr uint32_t kBox = 128 * 128;     // one 64-column box of 128 rows
  static constexpr uint32_t kX = 0;               // two X buffers
  static constexpr uint32_t kRing = 2 * kTile;    // two stages of (hi, lo)
  static constexpr uint32_t kStage = 2 * kTile;
  static constexpr uint32_t kNsq = kRing + 2 * kStage;  // 4 warps x 128 floats
  static constexpr uint32_t kBar = kNsq + 4 * kAsgChunk * 4;
  static constexpr int kXFull = 0, kXEmpty = 2, kFull = 4, kEmpty = 6, kAFull = 8, kAEmpty = 10, kFinal = 12,
                       kNumBars = 13;
  static constexpr uint32_t kMisc = kBar + kNumBars * 8;
  static constexpr uint32_t kAlloc = kMisc + 16 + 1024;
};

template <int D>
__global__ void __launch_bounds__(kAsgThreads, 1)
    cluster_assign_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_hi,
                          const __grid_constant__ CUtensorMap tm_lo, ClusterLaunch l, uint64_t timeout_ns,
                          int* status) {
  using namespace isa_dev;
  using L = AsgLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  auto bar = [&](int i) -> uint32_t { return base + L::kBar + 8u * static_cast<uint32_t>(i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tiles_per_head = (l.N + kAsgRows - 1) / kAsgRows;
  const int64_t n_tiles = static_cast<int64_t>(l.BH) * tiles_per_head;
  const int nch = l.Cpad / kAsgChunk;

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(L::kXFull + i), 1);
      mbar_init(bar(L::kXEmpty + i), 1);
      mbar_init(bar(L::kFull + i), 1);
      mbar_init(bar(L::kEmpty + i), 1);
      mbar_init(bar(L::kAFull + i), 1);
      mbar_init(bar(L::kAEmpty + i), 128);
    }
    mbar_init(bar(L::kFinal), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(smem_addr(tmem_slot), 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t item = 0, tc = 0, issued = 0, x_issued = 0;
      bool ok = true;
      for (int64_t t = blockIdx.x; t < n_tiles && ok; t += gridDim.x, ++tc) {
        const int bh = static_cast<int>(t / tiles_per_head);
        const int row = static_cast<int>(t - static_cast<int64_t>(bh) * tiles_per_head) * kAsgRows;
        const uint32_t xb = tc & 1u;
        if (!mbar_wait(bar(L::kXEmpty + xb), ((tc >> 1) & 1u) ^ 1u, abort_flag, timeout_ns)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(bar(L::kXFull + xb), L::kTile);
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(base + L::kX + xb * L::kTile + c * L::kBox, &tm_x, bar(L::kXFull + xb), c * 64, row, bh);
        ++x_issued;
        for (int j = 0; j < nch; ++j, ++item) {
          const uint32_t s = item & 1u;
          if (!mbar_wait(bar(L::kEmpty + s), ((item >> 1) & 1u) ^ 1u, abort_flag, timeout_ns)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar(L::kFull + s), L::kStage);
          const uint32_t dst = base + L::kRing + s * L::kStage;
#pragma unroll
          for (int c = 0; c < D / 64; ++c) {
            tma_load_3d(dst + c * L::kBox, &tm_hi, bar(L::kFull + s), c * 64, j * kAsgChunk, bh);
            tma_load_3d(dst + L::kTile + c * L::kBox, &tm_lo, bar(L::kFull + s), c * 64, j * kAsgChunk, bh);
          }
          ++issued;
        }
      }
      if (!ok || *abort_flag) {
        // let the copies already issued land before the CTA leaves
        const uint32_t first = issued > 2 ? issued - 2 : 0;
        for (uint32_t i = first; i < issued; ++i) {
          const uint64_t t0 = global_timer_ns();
          while (!mbar_try_wait(bar(L::kFull + (i & 1u)), (i >> 1) & 1u))
            if (global_timer_ns() - t0 > 200000000ull) break;
        }
        const uint32_t xfirst = x_issued > 2 ? x_issued - 2 : 0;
        for (uint32_t i = xfirst; i < x_issued; ++i) {
          const uint64_t t0 = global_timer_ns();
          while (!mbar_try_wait(bar(L::kXFull + (i & 1u)), (i >> 1) & 1u))
            if (global_timer_ns() - t0 > 200000000ull) break;
        }
      }
    }
  } else if (warp == 5) {
    // ----------------------------------------------------------------- MMA
    constexpr uint32_t idesc = idesc_bf16_f32(128, kAsgChunk, 0);
    const uint64_t dx = smem_desc_sw128(base + L::kX, 16, 1024);
    const uint64_t dr = smem_desc_sw128(base + L::kRing, 16, 1024);
    uint32_t item = 0, tc = 0;
    bool ok = true;
    for (int64_t t = blockIdx.x; t < n_tiles && ok; t += gridDim.x, ++tc) {
      const uint32_t xb = tc & 1u;
      if (!mbar_wait_warp(bar(L::kXFull + xb), (tc >> 1) & 1u, abort_flag, timeout_ns)) break;
      const uint64_t a0 = dx + ((xb * L::kTile) >> 4);
      for (int j = 0; j < nch; ++j, ++item) {
        const uint32_t s = item & 1u, ab = item & 1u;
        if (!mbar_wait_warp(bar(L::kFull + s), (item >> 1) & 1u, abort_flag, timeout_ns) ||
            !mbar_wait_warp(bar(L::kAEmpty + ab), ((item >> 1) & 1u) ^ 1u, abort_flag, timeout_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t b_hi = dr + ((s * L::kStage) >> 4), b_lo = b_hi + (L::kTile >> 4);
        const uint32_t d = tmem + ab * kAsgChunk;
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint64_t off = ((k >> 2) * L::kBox + (k & 3) * 32) >> 4;
          if (elect_one()) mma_ss(d, a0 + off, b_hi + off, idesc, k > 0 ? 1u : 0u);
          if (elect_one()) mma_ss(d, a0 + off, b_lo + off, idesc, 1u);
        }
        if (elect_one()) {
          tc_commit(bar(L::kEmpty + s));
          tc_commit(bar(L::kAFull + ab));
          if (j == nch - 1) tc_commit(bar(L::kXEmpty + xb));
        }
      }
    }
    if (elect_one()) tc_commit(bar(L::kFinal));
    __syncwarp();
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar(L::kFinal), 0))
      if (global_timer_ns() - t0 > 200000000ull) break;
  } else {
    // ------------------------------------------------------------ epilogue
    const int r = warp * 32 + lane;  // row of the tile == TMEM lane
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    float* nsq_s = reinterpret_cast<float*>(smem + L::kNsq) + warp * kAsgChunk;
    // this lane's four norms of an item's chunk, fetched one item ahead
    auto fetch = [&](int64_t t, int j) -> float4 {
      const int bh = static_cast<int>(t / tiles_per_head);
      return *reinterpret_cast<const float4*>(l.mu_nsq + static_cast<int64_t>(bh) * l.Cpad + j * kAsgChunk +
                                              4 * lane);
    };
    uint32_t item = 0;
    int64_t t = blockIdx.x;
    float4 nq = t < n_tiles ? fetch(t, 0) : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    bool ok = true;
    for (; t < n_tiles && ok; t += gridDim.x) {
      const int bh = static_cast<int>(t / tiles_per_head);
      const int row0 = static_cast<int>(t - static_cast<int64_t>(bh) * tiles_per_head) * kAsgRows;
      float best = INFINITY;
      int bi = 0;
      for (int j = 0; j < nch; ++j, ++item) {
        __syncwarp();
        *reinterpret_cast<float4*>(nsq_s + 4 * lane) = nq;
        __syncwarp();
        if (j + 1 < nch)
          nq = fetch(t, j + 1);
        else if (t + gridDim.x < n_tiles)
          nq = fetch(t + gridDim.x, 0);
        const uint32_t ab = item & 1u;
        if (!mbar_wait(bar(L::kAFull + ab), (item >> 1) & 1u, abort_flag, timeout_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t v[4][32];
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) tmem_ld32(lane_base + ab * kAsgChunk + 32 * cc, v[cc]);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(bar(L::kAEmpty + ab));
#pragma unroll
        for (int cc = 0; cc < 4; ++cc)
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            const float4 n4 = *reinterpret_cast<const float4*>(nsq_s + 32 * cc + e);
            const float nn[4] = {n4.x, n4.y, n4.z, n4.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const float dist = fmaf(-2.0f, __uint_as_float(v[cc][e + u]), nn[u]);
              if (dist < best) {
                best = dist;
                bi = j * kAsgChunk + 32 * cc + e + u;
              }
            }
          }
      }
      if (ok && row0 + r < l.N) l.labels[static_cast<int64_t>(bh) * l.N + row0 + r] = bi;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (tid == 0 && *abort_flag) atomicCAS(status, 0, kStatusTimeout);
  if (warp == 5) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// Stable counting sort of one head's labels, one CTA of W warps per (batch,
// head); warp w owns the contiguous rows [w seg, (w+1) seg):
//   count  each warp counts its rows into its own histogram row hist[w][c];
//   scan   per cluster, the column prefix over the warps gives each warp's
//          first position inside the cluster, and a block-wide exclusive
//          scan of the cluster totals gives the offsets (and the offsets of
//          the non-empty clusters: the query groups);
//   place  each warp walks its rows in ascending order, 32 at a time: lanes
//          with equal labels rank themselves by lane order
//          (__match_any_sync) and the lowest of them moves the warp's cursor.
// Rows keep their order inside a cluster because the warps' segments are
// ordered and each warp places its rows in order.  Labels are read
// 32 x kSortBatch at a time, a batch ahead of the one being processed.  A
// label outside [0, C) is skipped and sets the device-check status (its row
// then has no place in perm).
constexpr int kSortBatch = 8;
constexpr int kSortMaxWarps = 16;

__global__ void __launch_bounds__(kSortMaxWarps * 32) cluster_sort_kernel(ClusterLaunch l, int* status) {
  extern __shared__ __align__(16) int32_t hist[];  // [W][C]: counts, then cursors
  __shared__ int32_t red_rows[kSortMaxWarps], red_ne[kSortMaxWarps];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, W = blockDim.x >> 5;
  const int64_t bh = blockIdx.x;
  const int N = l.N, C = l.C;
  const int32_t* lab = l.labels + bh * N;
  const int seg = (N + W - 1) / W;
  const int s0 = min(N, warp * seg), s1 = min(N, s0 + seg);
  int32_t* my = hist + static_cast<int64_t>(warp) * C;
  for (int c = lane; c < C; c += 32) my[c] = 0;
  __syncwarp();
  auto load_batch = [&](int base, int (&v)[kSortBatch]) {
#pragma unroll
    for (int k = 0; k < kSortBatch; ++k) {
      const int r = base + 32 * k + lane;
      v[k] = r < s1 ? lab[r] : -1;
    }
  };
  constexpr int kStep = 32 * kSortBatch;
  bool bad = false;
  int v[kSortBatch], nx[kSortBatch];
  load_batch(s0, v);
  for (int base = s0; base < s1; base += kStep) {
    if (base + kStep < s1) load_batch(base + kStep, nx);
#pragma unroll
    for (int k = 0; k < kSortBatch; ++k) {
      if (v[k] >= 0 && v[k] < C) {
        atomicAdd(&my[v[k]], 1);
      } else if (base + 32 * k + lane < s1) {
        bad = true;
      }
    }
#pragma unroll
    for (int k = 0; k < kSortBatch; ++k) v[k] = nx[k];
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) atomicCAS(status, 0, kStatusDeviceCheck);
  __syncthreads();

  // scan: thread t owns clusters [c0, c1)
  const int T = blockDim.x;
  const int E = (C + T - 1) / T;
  const int c0 = min(C, tid * E), c1 = min(C, c0 + E);
  int rows_local = 0, ne_local = 0;
  for (int c = c0; c < c1; ++c) {
    int n = 0;
    for (int w = 0; w < W; ++w) n += hist[static_cast<int64_t>(w) * C + c];
    rows_local += n;
    ne_local += n > 0 ? 1 : 0;
  }
  int rows_incl = rows_local, ne_incl = ne_local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t0 = __shfl_up_sync(0xffffffffu, rows_incl, o);
    const int t1 = __shfl_up_sync(0xffffffffu, ne_incl, o);
    if (lane >= o) {
      rows_incl += t0;
      ne_incl += t1;
    }
  }
  if (lane == 31) {
    red_rows[warp] = rows_incl;
    red_ne[warp] = ne_incl;
  }
  __syncthreads();
  int rows_before = 0, ne_before = 0, rows_all = 0, ne_all = 0;
  for (int w = 0; w < W; ++w) {
    if (w < warp) {
      rows_before += red_rows[w];
      ne_before += red_ne[w];
    }
    rows_all += red_rows[w];
    ne_all += red_ne[w];
  }
  int run = rows_before + rows_incl - rows_local, g = ne_before + ne_incl - ne_local;
  int32_t* off = l.offsets + bh * (C + 1);
  int32_t* grp = l.groups ? l.groups + bh * (C + 1) : nullptr;
  for (int c = c0; c < c1; ++c) {
    int col = run;
    for (int w = 0; w < W; ++w) {
      int32_t& h = hist[static_cast<int64_t>(w) * C + c];
      const int x = h;
      h = col;
      col += x;
    }
    const int n = col - run;
    off[c] = run;
    if (grp && n > 0) grp[g++] = run;
    run = col;
  }
  if (tid == 0) {
    off[C] = rows_all;
    if (grp) grp[ne_all] = rows_all;
    if (l.n_groups) l.n_groups[bh] = ne_all;
  }
  __syncthreads();

  // place
  int32_t* pm = l.perm + bh * N;
  load_batch(s0, v);
  for (int base = s0; base < s1; base += kStep) {
    if (base + kStep < s1) load_batch(base + kStep, nx);
#pragma unroll
    for (int k = 0; k < kSortBatch; ++k) {
      const int c = (v[k] >= 0 && v[k] < C) ? v[k] : -1;
      const unsigned peers = __match_any_sync(0xffffffffu, c);
      const int rank = __popc(peers & ((1u << lane) - 1u));
      const int pos = c >= 0 ? my[c] + rank : 0;
      __syncwarp();
      if (c >= 0) {
        pm[pos] = base + 32 * k + lane;
        if (rank == 0) my[c] += __popc(peers);
      }
      __syncwarp();
    }
#pragma unroll
    for (int k = 0; k < kSortBatch; ++k) v[k] = nx[k];
  }
}

// mu_c = mean of cluster c's rows in permutation order (fp32, a fixed order,
// so the result does not depend on scheduling); an empty cluster keeps its
// centroid.  One warp per centroid, 16 row loads in flight; the hi / lo /
// norm operands of the next assignment are written too.
template <int D>
__global__ void __launch_bounds__(kPrepWarps * 32) cluster_update_kernel(ClusterLaunch l) {
  constexpr int PER = D / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x * kPrepWarps + warp;
  const int64_t bh = blockIdx.y;
  if (c >= l.C) return;
  const int32_t* off = l.offsets + bh * (l.C + 1);
  const int s = off[c], e = off[c + 1];
  const int32_t* pm = l.perm + bh * l.N;
  const uint16_t* xb = static_cast<const uint16_t*>(l.x) + bh * l.N * D + lane * PER;
  float* mu = l.mu + (bh * l.C + c) * D + lane * PER;
  float v[PER];
  if (e > s) {
    float acc[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) acc[i] = 0.0f;
    // 32 positions at a time: lane k loads perm[b0 + k], then the rows go
    // 16 loads in flight at a time and are added in position order
    constexpr int kU = 16;
    for (int b0 = s; b0 < e; b0 += 32) {
      const int n = min(32, e - b0);
      const int my_r = lane < n ? pm[b0 + lane] : 0;
      for (int k0 = 0; k0 < n; k0 += kU) {
        float f[kU][PER];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          const int r = __shfl_sync(0xffffffffu, my_r, (k0 + u) & 31);
          const uint16_t* p = xb + static_cast<int64_t>(r) * D;
          if constexpr (PER == 4) {
            const uint2 w = k0 + u < n ? *reinterpret_cast<const uint2*>(p) : make_uint2(0u, 0u);
            f[u][0] = bf16f(w.x & 0xFFFF);
            f[u][1] = bf16f(w.x >> 16);
            f[u][2] = bf16f(w.y & 0xFFFF);
            f[u][3] = bf16f(w.y >> 16);
          } else {
            const uint32_t w = k0 + u < n ? *reinterpret_cast<const uint32_t*>(p) : 0u;
            f[u][0] = bf16f(w & 0xFFFF);
            f[u][1] = bf16f(w >> 16);
          }
        }
#pragma unroll
        for (int u = 0; u < kU; ++u)
          if (k0 + u < n) {
#pragma unroll
            for (int q = 0; q < PER; ++q) acc[q] += f[u][q];
          }
      }
    }
    const float inv = 1.0f / static_cast<float>(e - s);
#pragma unroll
    for (int k = 0; k < PER; ++k) {
      v[k] = acc[k] * inv;
      mu[k] = v[k];
    }
  } else {
#pragma unroll
    for (int k = 0; k < PER; ++k) v[k] = mu[k];
  }
  write_prep<D>(l, bh, c, v, true);
}

// out[row i] = x[row perm[i]] (gather) or out[row perm[i]] = x[row i]
// (scatter, the inverse), rows of D bf16 values, one 16-byte vector per
// thread.  An index outside [0, N) is skipped and sets the device-check status.
__global__ void __launch_bounds__(256) permute_rows_kernel(const uint16_t* __restrict__ x,
                                                           const int32_t* __restrict__ perm, int64_t BH, int N, int D,
                                                           int inverse, uint16_t* __restrict__ out, int* status) {
  const int vpr = D / 8;
  const int64_t total = BH * N * vpr;
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < total;
       t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t row = t / vpr;
    const int v = static_cast<int>(t - row * vpr);
    const int64_t bh = row / N;
    const int i = static_cast<int>(row - bh * N);
    const int p = perm[row];
    if (p < 0 || p >= N) {
      if (v == 0) atomicCAS(status, 0, kStatusDeviceCheck);
      continue;
    }
    const int src = inverse ? i : p, dst = inverse ? p : i;
    const uint4 w = *reinterpret_cast<const uint4*>(x + ((bh * N + src) * D + v * 8));
    *reinterpret_cast<uint4*>(out + ((bh * N + dst) * D + v * 8)) = w;
  }
}

template <int D>
int launch_assign_d(const ClusterLaunch& l, int num_sms, uint64_t timeout_ns, int* status, cudaStream_t stream) {
  using L = AsgLayout<D>;
  CUtensorMap tx, thi, tlo;
  if (!make_bf16_map(&tx, l.x, l.BH, l.N, D, 128) || !make_bf16_map(&thi, l.mu_hi, l.BH, l.Cpad, D, 128) ||
      !make_bf16_map(&tlo, l.mu_lo, l.BH, l.Cpad, D, 128))
    return -1;
  {
    const cudaError_t e =
        ensure_smem_attr(reinterpret_cast<const void*>(cluster_assign_kernel<D>), static_cast<int>(L::kAlloc));
    if (e != cudaSuccess) return static_cast<int>(e);
  }
  const int64_t n_tiles = static_cast<int64_t>(l.BH) * ((l.N + kAsgRows - 1) / kAsgRows);
  const int grid = static_cast<int>(n_tiles < num_sms ? n_tiles : num_sms);
  cluster_assign_kernel<D><<<grid, kAsgThreads, L::kAlloc, stream>>>(tx, thi, tlo, l, timeout_ns, status);
  return static_cast<int>(cudaGetLastError());
}

}  // namespace

int launch_cluster_prep(const ClusterLaunch& l, cudaStream_t stream) {
  const dim3 grid((l.Cpad + kPrepWarps - 1) / kPrepWarps, l.BH);
  if (l.D == 128)
    cluster_prep_kernel<128><<<grid, kPrepWarps * 32, 0, stream>>>(l);
  else
    cluster_prep_kernel<64><<<grid, kPrepWarps * 32, 0, stream>>>(l);
  return static_cast<int>(cudaGetLastError());
}

int launch_cluster_init(const ClusterLaunch& l, cudaStream_t stream) {
  const dim3 grid((l.C + kPrepWarps - 1) / kPrepWarps, l.BH);
  if (l.D == 128)
    cluster_init_kernel<128><<<grid, kPrepWarps * 32, 0, stream>>>(l);
  else
    cluster_init_kernel<64><<<grid, kPrepWarps * 32, 0, stream>>>(l);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return static_cast<int>(e);
  return launch_cluster_prep(l, stream);
}

int launch_cluster_assign(const ClusterLaunch& l, int num_sms, uint64_t timeout_ns, int* status,
                          cudaStream_t stream) {
  const uint64_t t = timeout_ns ? timeout_ns : kWaitTimeoutNs;
  return l.D == 128 ? launch_assign_d<128>(l, num_sms, t, status, stream)
                    : launch_assign_d<64>(l, num_sms, t, status, stream);
}

int launch_cluster_sort(const ClusterLaunch& l, int* status, cudaStream_t stream) {
  // as many warps per head as keep the per-warp histograms within 64 KB
  int W = 16384 / (l.C > 0 ? l.C : 1);
  W = W < 1 ? 1 : (W > kSortMaxWarps ? kSortMaxWarps : W);
  const size_t smem = static_cast<size_t>(W) * l.C * 4;
  if (smem > 48 * 1024) {
    const cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(cluster_sort_kernel), 64 * 1024);
    if (e != cudaSuccess) return static_cast<int>(e);
  }
  cluster_sort_kernel<<<l.BH, W * 32, smem, stream>>>(l, status);
  return static_cast<int>(cudaGetLastError());
}

int launch_cluster_update(const ClusterLaunch& l, cudaStream_t stream) {
  const dim3 grid((l.C + kPrepWarps - 1) / kPrepWarps, l.BH);
  if (l.D == 128)
    cluster_update_kernel<128><<<grid, kPrepWarps * 32, 0, stream>>>(l);
  else
    cluster_update_kernel<64><<<grid, kPrepWarps * 32, 0, stream>>>(l);
  return static_cast<int>(cudaGetLastError());
}

int launch_permute_rows(const void* x, const int32_t* perm, int BH, int N, int D, bool inverse, void* out, int* status,
                        int num_sms, cudaStream_t stream) {
  const int64_t total = static_cast<int64_t>(BH) * N * (D / 8);
  const int64_t want = (total + 255) / 256;
  const int64_t cap = static_cast<int64_t>(num_sms) * 8;
  const int grid = static_cast<int>(want < cap ? want : cap);
  permute_rows_kernel<<<grid > 0 ? grid : 1, 256, 0, stream>>>(static_cast<const uint16_t*>(x), perm, BH, N, D,
                                                              inverse ? 1 : 0, static_cast<uint16_t*>(out), status);
  return static_cast<int>(cudaGetLastError());
}

}  // namespace isa_impl
