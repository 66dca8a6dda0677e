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
//           the lower c; the dot products run on tensor cores (mma.sync
//           m16n8k16) with x exact in bf16 and mu split into bf16 hi + lo
//           parts (relative error 2^-16), two products per tile;
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

namespace isa_impl {
namespace {

__device__ __forceinline__ float bf16f(uint16_t h) { return __uint_as_float(static_cast<uint32_t>(h) << 16); }

constexpr int kAsgThreads = 128;  // 4 warps x 32 rows
constexpr int kAsgRows = 128;
constexpr int kAsgChunk = 64;     // centroids per shared-memory stage
constexpr int kPrepWarps = 8;

template <int D>
struct AsgLayout {
  static constexpr int XS = D + 8;  // padded row (elements): ldmatrix rows land in distinct banks
  static constexpr uint32_t kX = 0;
  static constexpr uint32_t kXBytes = kAsgRows * XS * 2;
  static constexpr uint32_t kStageBytes = 2 * kAsgChunk * XS * 2;  // hi rows, then lo rows
  static constexpr uint32_t kC = kXBytes;
  static constexpr uint32_t kN = kC + 2 * kStageBytes;
  static constexpr uint32_t kAlloc = kN + 2 * kAsgChunk * 4;
};

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

// Nearest centroid of 128 rows per CTA.  The rows sit in shared memory and,
// as mma A fragments, in registers (two 16-row tiles per warp); centroids
// stream through a two-stage cp.async ring 64 at a time.  Within a lane the
// candidates come in ascending c and a strict compare keeps the first
// minimum; across the quad, equal distances go to the lower c.
template <int D>
__global__ void __launch_bounds__(kAsgThreads) cluster_assign_kernel(ClusterLaunch l) {
  using namespace isa_dev;
  using L = AsgLayout<D>;
  constexpr int XS = L::XS, KSTEPS = D / 16;
  extern __shared__ __align__(16) uint8_t sm[];
  const uint32_t sbase = smem_addr(sm);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gq = lane >> 2, tq = lane & 3;
  const int64_t bh = blockIdx.y;
  const int r0 = blockIdx.x * kAsgRows;
  const int rows = min(kAsgRows, l.N - r0);
  const uint16_t* xg = static_cast<const uint16_t*>(l.x) + (bh * l.N + r0) * D;
  for (int i = tid; i < kAsgRows * (D / 8); i += kAsgThreads) {
    const int r = i / (D / 8), c16 = i - r * (D / 8);
    const bool in = r < rows;
    cp_async16_zfill(sbase + L::kX + 2u * (r * XS + c16 * 8), in ? xg + static_cast<int64_t>(r) * D + c16 * 8 : xg,
                     in ? 16u : 0u);
  }
  const uint16_t* hig = l.mu_hi + bh * l.Cpad * D;
  const uint16_t* lowg = l.mu_lo + bh * l.Cpad * D;
  const float* nsg = l.mu_nsq + bh * l.Cpad;
  auto load_stage = [&](int ch, int st) {
    const uint32_t dst = sbase + L::kC + st * L::kStageBytes;
    for (int i = tid; i < kAsgChunk * (D / 8); i += kAsgThreads) {
      const int r = i / (D / 8), c16 = i - r * (D / 8);
      const int64_t src = static_cast<int64_t>(ch * kAsgChunk + r) * D + c16 * 8;
      cp_async16(dst + 2u * (r * XS + c16 * 8), hig + src);
      cp_async16(dst + 2u * ((kAsgChunk + r) * XS + c16 * 8), lowg + src);
    }
    if (tid < kAsgChunk / 4) cp_async16(sbase + L::kN + st * kAsgChunk * 4 + tid * 16, nsg + ch * kAsgChunk + tid * 4);
  };
  const int n_chunks = l.Cpad / kAsgChunk;
  load_stage(0, 0);
  cp_async_commit();
  // ldmatrix lane addresses: A tile (rows, k) and a pair of B n-tiles
  // (matrices: n 0-7 k 0-7, n 0-7 k 8-15, n 8-15 k 0-7, n 8-15 k 8-15)
  const int a_row = (lane & 7) + ((lane >> 3) & 1) * 8, a_col = (lane >> 4) * 8;
  const int b_row = (lane & 7) + (lane >> 4) * 8, b_col = ((lane >> 3) & 1) * 8;
  uint32_t a[2][KSTEPS][4];
  float best[2][2];
  int bi[2][2];
#pragma unroll
  for (int t = 0; t < 2; ++t)
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      best[t][hh] = INFINITY;
      bi[t][hh] = 0;
    }
  for (int ch = 0; ch < n_chunks; ++ch) {
    const int st = ch & 1;
    if (ch + 1 < n_chunks) {
      load_stage(ch + 1, st ^ 1);
      cp_async_commit();
      cp_async_wait_group<1>();
    } else {
      cp_async_wait_group<0>();
    }
    __syncthreads();
    if (ch == 0) {
#pragma unroll
      for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int ks = 0; ks < KSTEPS; ++ks)
          ldsm_x4(a[t][ks], sbase + L::kX + 2u * ((32 * warp + 16 * t + a_row) * XS + ks * 16 + a_col));
    }
    const uint32_t hi_s = sbase + L::kC + st * L::kStageBytes, lo_s = hi_s + kAsgChunk * XS * 2;
    const float* ns = reinterpret_cast<const float*>(sm + L::kN) + st * kAsgChunk;
#pragma unroll 1
    for (int np = 0; np < kAsgChunk / 16; ++np) {
      float acc[2][2][4];
#pragma unroll
      for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
          for (int k = 0; k < 4; ++k) acc[t][j][k] = 0.0f;
#pragma unroll
      for (int ks = 0; ks < KSTEPS; ++ks) {
        uint32_t bh4[4], bl4[4];
        const uint32_t off = 2u * ((np * 16 + b_row) * XS + ks * 16 + b_col);
        ldsm_x4(bh4, hi_s + off);
        ldsm_x4(bl4, lo_s + off);
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
          for (int j = 0; j < 2; ++j) mma_16816(acc[t][j], a[t][ks], bh4[2 * j], bh4[2 * j + 1]);
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
          for (int j = 0; j < 2; ++j) mma_16816(acc[t][j], a[t][ks], bl4[2 * j], bl4[2 * j + 1]);
      }
#pragma unroll
      for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int cl = np * 16 + j * 8 + 2 * tq + e;
          const float nsq = ns[cl];
          const int c = ch * kAsgChunk + cl;
#pragma unroll
          for (int t = 0; t < 2; ++t)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              const float dist = nsq - 2.0f * acc[t][j][2 * hh + e];
              if (dist < best[t][hh]) {
                best[t][hh] = dist;
                bi[t][hh] = c;
              }
            }
        }
    }
    __syncthreads();  // every warp is done with this stage before it is refilled
  }
#pragma unroll
  for (int t = 0; t < 2; ++t)
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      float b = best[t][hh];
      int i = bi[t][hh];
#pragma unroll
      for (int o = 1; o <= 2; o <<= 1) {
        const float ob = __shfl_xor_sync(0xffffffffu, b, o);
        const int oi = __shfl_xor_sync(0xffffffffu, i, o);
        if (ob < b || (ob == b && oi < i)) {
          b = ob;
          i = oi;
        }
      }
      const int r = 32 * warp + 16 * t + gq + 8 * hh;
      if (tq == 0 && r < rows) l.labels[bh * l.N + r0 + r] = i;
    }
}

// Stable counting sort of one head's labels, one warp per (batch, head):
// histogram in shared memory, an exclusive scan into the offsets (and the
// offsets of the non-empty clusters: the query groups), then the rows in
// ascending order, 32 at a time: lanes with equal labels rank themselves by
// lane order (__match_any_sync) and the lowest of them moves the cluster's
// cursor.  Labels are read 32 x kSortBatch at a time, so that their loads
// are in flight together.  A label outside [0, C) is skipped and sets the
// device-check status (its row then has no place in perm).
constexpr int kSortBatch = 16;

__global__ void __launch_bounds__(32) cluster_sort_kernel(ClusterLaunch l, int* status) {
  extern __shared__ __align__(16) int32_t cur[];  // [C]: counts, then cursors
  const int lane = threadIdx.x;
  const int64_t bh = blockIdx.x;
  const int N = l.N, C = l.C;
  const int32_t* lab = l.labels + bh * N;
  for (int c = lane; c < C; c += 32) cur[c] = 0;
  __syncwarp();
  bool bad = false;
  for (int base = 0; base < N; base += 32 * kSortBatch) {
    int v[kSortBatch];
#pragma unroll
    for (int k = 0; k < kSortBatch; ++k) {
      const int r = base + 32 * k + lane;
      v[k] = r < N ? lab[r] : -1;
    }
#pragma unroll
    for (int k = 0; k < kSortBatch; ++k) {
      if (v[k] >= 0 && v[k] < C) {
        atomicAdd(&cur[v[k]], 1);
      } else if (base + 32 * k + lane < N) {
        bad = true;
      }
    }
  }
  __syncwarp();
  // lane owns clusters [c0, c1)
  const int E = (C + 31) / 32;
  const int c0 = min(C, lane * E), c1 = min(C, c0 + E);
  int rows_local = 0, ne_local = 0;
  for (int c = c0; c < c1; ++c) {
    rows_local += cur[c];
    ne_local += cur[c] > 0 ? 1 : 0;
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
  int run = rows_incl - rows_local, g = ne_incl - ne_local;
  int32_t* off = l.offsets + bh * (C + 1);
  int32_t* grp = l.groups ? l.groups + bh * (C + 1) : nullptr;
  for (int c = c0; c < c1; ++c) {
    const int n = cur[c];
    off[c] = run;
    if (grp && n > 0) grp[g++] = run;
    cur[c] = run;
    run += n;
  }
  if (lane == 31) {
    off[C] = rows_incl;
    if (grp) grp[ne_incl] = rows_incl;
    if (l.n_groups) l.n_groups[bh] = ne_incl;
  }
  __syncwarp();
  int32_t* pm = l.perm + bh * N;
  for (int base = 0; base < N; base += 32 * kSortBatch) {
    int v[kSortBatch];
#pragma unroll
    for (int k = 0; k < kSortBatch; ++k) {
      const int r = base + 32 * k + lane;
      const int c = r < N ? lab[r] : -1;
      v[k] = (c >= 0 && c < C) ? c : -1;
    }
#pragma unroll
    for (int k = 0; k < kSortBatch; ++k) {
      const int c = v[k];
      const unsigned peers = __match_any_sync(0xffffffffu, c);
      const int rank = __popc(peers & ((1u << lane) - 1u));
      const int pos = c >= 0 ? cur[c] + rank : 0;
      __syncwarp();
      if (c >= 0) {
        pm[pos] = base + 32 * k + lane;
        if (rank == 0) cur[c] += __popc(peers);
      }
      __syncwarp();
    }
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) atomicCAS(status, 0, kStatusDeviceCheck);
}

// mu_c = mean of cluster c's rows in permutation order (fp32, a fixed order,
// so the result does not depend on scheduling); an empty cluster keeps its
// centroid.  One warp per centroid; the hi / lo / norm operands of the next
// assignment are written too.
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
    auto add_row = [&](int r) {
      const uint16_t* p = xb + static_cast<int64_t>(r) * D;
      if constexpr (PER == 4) {
        const uint2 w = *reinterpret_cast<const uint2*>(p);
        acc[0] += bf16f(w.x & 0xFFFF);
        acc[1] += bf16f(w.x >> 16);
        acc[2] += bf16f(w.y & 0xFFFF);
        acc[3] += bf16f(w.y >> 16);
      } else {
        const uint32_t w = *reinterpret_cast<const uint32_t*>(p);
        acc[0] += bf16f(w & 0xFFFF);
        acc[1] += bf16f(w >> 16);
      }
    };
    int i = s;
    for (; i + 4 <= e; i += 4) {
      // the four rows' loads are issued before the first add
      const int ra = pm[i], rb = pm[i + 1], rc = pm[i + 2], rd = pm[i + 3];
      if constexpr (PER == 4) {
        const uint2 wa = *reinterpret_cast<const uint2*>(xb + static_cast<int64_t>(ra) * D);
        const uint2 wb = *reinterpret_cast<const uint2*>(xb + static_cast<int64_t>(rb) * D);
        const uint2 wc = *reinterpret_cast<const uint2*>(xb + static_cast<int64_t>(rc) * D);
        const uint2 wd = *reinterpret_cast<const uint2*>(xb + static_cast<int64_t>(rd) * D);
        const uint2 w4[4] = {wa, wb, wc, wd};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          acc[0] += bf16f(w4[k].x & 0xFFFF);
          acc[1] += bf16f(w4[k].x >> 16);
          acc[2] += bf16f(w4[k].y & 0xFFFF);
          acc[3] += bf16f(w4[k].y >> 16);
        }
      } else {
        add_row(ra);
        add_row(rb);
        add_row(rc);
        add_row(rd);
      }
    }
    for (; i < e; ++i) add_row(pm[i]);
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
int launch_assign_d(const ClusterLaunch& l, cudaStream_t stream) {
  using L = AsgLayout<D>;
  static bool attr = false;
  if (!attr) {
    const cudaError_t e = cudaFuncSetAttribute(cluster_assign_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(L::kAlloc));
    if (e != cudaSuccess) return static_cast<int>(e);
    attr = true;
  }
  cluster_assign_kernel<D><<<dim3((l.N + kAsgRows - 1) / kAsgRows, l.BH), kAsgThreads, L::kAlloc, stream>>>(l);
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

int launch_cluster_assign(const ClusterLaunch& l, cudaStream_t stream) {
  return l.D == 128 ? launch_assign_d<128>(l, stream) : launch_assign_d<64>(l, stream);
}

int launch_cluster_sort(const ClusterLaunch& l, int* status, cudaStream_t stream) {
  const size_t smem = static_cast<size_t>(l.C) * 4;
  if (smem > 48 * 1024) {
    const cudaError_t e =
        cudaFuncSetAttribute(cluster_sort_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return static_cast<int>(e);
  }
  cluster_sort_kernel<<<l.BH, 32, smem, stream>>>(l, status);
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
