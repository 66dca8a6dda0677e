// IBCS block scorer.
//
// "AB-Attention: Accurate Block Attention for Accelerating Video Diffusion
// Transformers", Intra-Block Clustering Selector: similar queries are
// grouped only within each query block, each group gets a representative and
// a weight equal to its size, and the representatives score small key blocks
// without reordering tokens.  Key blocks are summarised by their means.
//
// Kernels:
//   key_means_kernel  kbar_b = mean of the valid rows of key block b, stored
//                     as a bf16 hi + lo pair;
//   kmeans_tc_kernel  (d = 128, groups of at most 128 rows) the k-means on
//                     tcgen05, one group per set of four warps; with C <= 8
//                     it also computes the key means in extra warps, in
//                     place of key_means_kernel;
//   kmeans_warp_kernel  per (batch*head, group), one warp: Lloyd's
//                     k-means, centroids initialised at rows floor(c n / C),
//                     `iters` rounds of nearest-centroid assignment (squared
//                     distance, ties to the lower c) and mean update; rows
//                     stream through shared memory 128 at a time;
//   mass_kernel       per (batch*head, 128 / C' groups): logits
//                     l = scale mu_c . kbar_b + ln L_b, a first pass for the
//                     per-centroid softmax max and sum over all key blocks, a
//                     second pass for mass_b = sum_c n_c exp(l - max_c) / sum_c.

#include <cuda_bf16.h>

#include <cstdint>

#include "isa_internal.h"
#include "mma_sync.cuh"
#include "ptx.cuh"
#include "tmap.h"

namespace isa_impl {
namespace {

constexpr int kScoreThreads = 256;
constexpr int kChunkRows = 128;

__device__ __forceinline__ float bf16_to_f(uint16_t h) { return __uint_as_float(static_cast<uint32_t>(h) << 16); }

// ------------------------------------------------------------ key means
// kbar_b = mean of the valid rows of key block b, written as a bf16 hi + lo
// pair (hi = bf16(kbar), lo = bf16(kbar - hi)) for the tensor-core mass product.
// One warp, key block b of (batch*head) bh; lane l sums dimensions
// PER l .. PER l + PER - 1 over the block's rows in order.
template <int D>
__device__ __forceinline__ void key_mean_block(const uint16_t* __restrict__ k, int N, int Bk, int nK, int64_t bh,
                                               int b, int lane, uint16_t* __restrict__ kbar_hi,
                                               uint16_t* __restrict__ kbar_lo) {
  using namespace isa_dev;
  constexpr int PER = D / 32;
  const int r0 = b * Bk, r1 = min(N, r0 + Bk);
  float acc[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) acc[i] = 0.0f;
  const uint16_t* base = k + (bh * N) * D + lane * PER;
  for (int r = r0; r < r1; ++r) {
    const uint16_t* p = base + static_cast<int64_t>(r) * D;
    if constexpr (PER == 4) {
      const uint2 v = *reinterpret_cast<const uint2*>(p);
      acc[0] += bf16_to_f(v.x & 0xFFFF);
      acc[1] += bf16_to_f(v.x >> 16);
      acc[2] += bf16_to_f(v.y & 0xFFFF);
      acc[3] += bf16_to_f(v.y >> 16);
    } else {
      const uint32_t v = *reinterpret_cast<const uint32_t*>(p);
      acc[0] += bf16_to_f(v & 0xFFFF);
      acc[1] += bf16_to_f(v >> 16);
    }
  }
  const float inv = 1.0f / static_cast<float>(r1 - r0);
  const int64_t o = (bh * nK + b) * D + lane * PER;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const float m = acc[i] * inv;
    const uint16_t hi = bf16_bits_rn(m);
    kbar_hi[o + i] = hi;
    kbar_lo[o + i] = bf16_bits_rn(m - bf16_bits_to_f(hi));
  }
}

template <int D>
__global__ void __launch_bounds__(kScoreThreads) key_means_kernel(const uint16_t* __restrict__ k, int N, int Bk,
                                                                  int nK, uint16_t* __restrict__ kbar_hi,
                                                                  uint16_t* __restrict__ kbar_lo) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.x * (kScoreThreads / 32) + warp;
  if (b >= nK) return;
  key_mean_block<D>(k, N, Bk, nK, blockIdx.y, b, lane, kbar_hi, kbar_lo);
}

// The key blocks a fused k-means launch left (see kmeans_tc_kernel): each warp
// takes one block at a time from *kb_next, until all BH nK are taken.
template <int D>
__global__ void __launch_bounds__(kScoreThreads) key_means_rest_kernel(const uint16_t* __restrict__ k, int N,
                                                                       int Bk, int nK, int n_blk,
                                                                       uint16_t* __restrict__ kbar_hi,
                                                                       uint16_t* __restrict__ kbar_lo,
                                                                       uint32_t* __restrict__ kb_next) {
  const int lane = threadIdx.x & 31;
  for (;;) {
    int b = 0;
    if (lane == 0) b = static_cast<int>(atomicAdd(kb_next, 1u));
    b = __shfl_sync(0xffffffffu, b, 0);
    if (b >= n_blk) return;
    key_mean_block<D>(k, N, Bk, nK, b / nK, b % nK, lane, kbar_hi, kbar_lo);
  }
}

// ---------------------------------------------- k-means, one warp per group
// Rows stream through the warp's shared-memory buffer 128 at a time (a group
// of <= 128 rows is loaded once), padded to D + 8 elements so that ldmatrix
// reads are free of bank conflicts.
// Assignment: dist_c = |mu_c|^2 - 2 x.mu_c (|x|^2 is common to all c) with the
// dots on tensor cores: x is exact in bf16 and mu_c is split into bf16
// hi + lo parts (relative error 2^-18), two mma.sync per 16x8x16 tile.
// Update: the cluster sums are a one-hot product (assignment^T x) on tensor
// cores, exact products accumulated in fp32; mu_c = sum_c / n_c.
// Every step of a group runs in one warp, with no block-wide barriers:
//   * the lane holding row gq of an mma.sync C tile also holds, in the B
//     fragment layout, dimensions 16 ks + 2 tq + {0, 1, 8, 9} of centroid
//     gq (and gq + 8): the cluster sums come out of the one-hot product in
//     exactly the registers the next round's distance products read, so the
//     centroids never leave registers;
//   * the count of each cluster is the sum over an extra column of ones
//     stored beside every valid row (a row past the group's end holds 0);
//   * rows stream through the warp's shared-memory buffer 128 at a time by
//     cp.async.
constexpr int kKmWarps = 6;

template <int D>
struct KmLayout {
  static constexpr int XS = D + 8;  // padded row (elements); column D holds 1.0 for a valid row
  static constexpr uint32_t kXBytes = kChunkRows * XS * 2;
  static constexpr uint32_t kWarpBytes = kXBytes + kChunkRows * 4;  // + the chunk's assignments
  static constexpr uint32_t kAlloc = kKmWarps * kWarpBytes;
};

template <int D, int NTC>
__global__ void __launch_bounds__(kKmWarps * 32) kmeans_warp_kernel(const uint16_t* __restrict__ q, int BH, int N,
                                                                    int G, int q_block,
                                                                    const int32_t* __restrict__ off, int C,
                                                                    int iters, float* __restrict__ centroids,
                                                                    int32_t* __restrict__ counts, int min_rows,
                                                                    int* status) {
  using namespace isa_dev;
  using L = KmLayout<D>;
  constexpr int XS = L::XS;
  constexpr int KSTEPS = D / 16;  // k-steps of the distance products
  constexpr int NTS = D / 8 + 1;  // n-tiles of the cluster sums; the last one holds the counts
  extern __shared__ __align__(16) uint8_t sm[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gq = lane >> 2, tq = lane & 3;
  uint16_t* xs = reinterpret_cast<uint16_t*>(sm + warp * L::kWarpBytes);
  int* assign = reinterpret_cast<int*>(sm + warp * L::kWarpBytes + L::kXBytes);
  const uint32_t xs_base = smem_addr(xs);
  // ldmatrix row address of this lane: x4 A tile at (row0, col0); x4 trans B
  // tile from x rows: matrices (k 0-7, n 0-7), (k 8-15, n 0-7), (k 0-7, n 8-15), (k 8-15, n 8-15)
  const int a_row = (lane & 7) + ((lane >> 3) & 1) * 8, a_col = (lane >> 4) * 8;
  const int t_row = (lane & 7) + ((lane >> 3) & 1) * 8, t_col = (lane >> 4) * 8;
  const int64_t n_items = static_cast<int64_t>(BH) * G;
  for (int64_t item = static_cast<int64_t>(blockIdx.x) * kKmWarps + warp; item < n_items;
       item += static_cast<int64_t>(gridDim.x) * kKmWarps) {
    const int64_t bh = item / G;
    const int g = static_cast<int>(item - bh * G);
    int r0, r1;
    if (off) {
      r0 = off[g];
      r1 = off[g + 1];
      if (r0 < 0 || r1 > N || r1 <= r0) {  // malformed offsets: leave an empty group
        if (lane == 0) atomicCAS(status, 0, kStatusDeviceCheck);
        r1 = r0 = 0;
      }
    } else {
      r0 = g * q_block;
      r1 = min(N, r0 + q_block);
    }
    const int n = r1 - r0;
    if (n <= min_rows) continue;  // the tensor-core kernel runs the groups of at most min_rows rows
    const uint16_t* qg = q + (bh * N + r0) * D;
    // rows [cs, cs + rc) of the group into the warp's buffer (zero past rc),
    // with the column of ones beside each valid row
    auto load_chunk = [&](int cs, int rc) {
      __syncwarp();  // every lane is done with the previous rows
#pragma unroll 8
      for (int k2 = 0; k2 < kChunkRows * (D / 8) / 32; ++k2) {
        const int i = lane + 32 * k2;
        const int r = i / (D / 8), c16 = i - r * (D / 8);
        const bool in = r < rc;
        const uint16_t* src = in ? qg + static_cast<int64_t>(cs + r) * D + c16 * 8 : qg;
        cp_async16_zfill(xs_base + 2u * (r * XS + c16 * 8), src, in ? 16u : 0u);
      }
      for (int r = lane; r < kChunkRows; r += 32)
        *reinterpret_cast<uint4*>(xs + r * XS + D) = make_uint4(r < rc ? 0x3F80u : 0u, 0u, 0u, 0u);
      cp_async_wait_all();
      __syncwarp();
    };
    // a group of at most 128 rows is loaded once, before the centroids are
    // initialised from it
    const bool one_chunk = n <= kChunkRows;
    if (one_chunk) load_chunk(0, n);
    // this lane's dimensions of centroids gq (+ 8), initialised at rows
    // floor(c n / C)
    float mu[NTC][KSTEPS][4];
#pragma unroll
    for (int h = 0; h < NTC; ++h) {
      const int c = gq + 8 * h;
      const int r = (c < C && n > 0) ? static_cast<int>((static_cast<int64_t>(c) * n) / C) : -1;
#pragma unroll
      for (int ks = 0; ks < KSTEPS; ++ks)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int dim = 16 * ks + 2 * tq + (e & 1) + 8 * (e >> 1);
          mu[h][ks][e] = r < 0 ? 0.0f
                         : one_chunk ? bf16_to_f(xs[r * XS + dim])
                                     : bf16_to_f(qg[static_cast<int64_t>(r) * D + dim]);
        }
    }
    int cnt[NTC];
#pragma unroll
    for (int h = 0; h < NTC; ++h) cnt[h] = 0;
    for (int it = 0; it < iters; ++it) {
      // centroids as bf16 hi + lo B fragments, and |mu_c|^2
      uint32_t bhi[NTC][KSTEPS][2], blo[NTC][KSTEPS][2];
      float nsq[NTC];
#pragma unroll
      for (int h = 0; h < NTC; ++h) {
        float acc = 0.0f;
#pragma unroll
        for (int ks = 0; ks < KSTEPS; ++ks)
#pragma unroll
          for (int p = 0; p < 2; ++p) {
            const float x0 = mu[h][ks][2 * p], x1 = mu[h][ks][2 * p + 1];
            const uint32_t hi = pack_bf16x2(x0, x1);
            const float h0 = __uint_as_float(hi << 16), h1 = __uint_as_float(hi & 0xFFFF0000u);
            bhi[h][ks][p] = hi;
            blo[h][ks][p] = pack_bf16x2(x0 - h0, x1 - h1);
            acc = fmaf(x0, x0, acc);
            acc = fmaf(x1, x1, acc);
          }
        acc += __shfl_xor_sync(0xffffffffu, acc, 1);
        acc += __shfl_xor_sync(0xffffffffu, acc, 2);
        nsq[h] = acc;
      }
      // |mu|^2 of the two centroids (columns 2 tq, 2 tq + 1) of each n-tile
      float msq[NTC][2];
#pragma unroll
      for (int nt = 0; nt < NTC; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) msq[nt][e] = __shfl_sync(0xffffffffu, nsq[nt], 4 * (2 * tq + e));
      float sums[NTS][4];
#pragma unroll
      for (int i = 0; i < NTS; ++i)
#pragma unroll
        for (int k = 0; k < 4; ++k) sums[i][k] = 0.0f;
      for (int cs = 0; cs < n; cs += kChunkRows) {
        const int rc = min(kChunkRows, n - cs);
        if (!one_chunk) load_chunk(cs, rc);
        // assignment: dist_c = |mu_c|^2 - 2 x.mu_c; argmin over c (ties to the
        // lower c) of rows gq and gq + 8 of row tile rt
        auto pick = [&](int rt, const float (&acc)[NTC][4]) {
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            float best = INFINITY;
            int bi = 0;
#pragma unroll
            for (int nt = 0; nt < NTC; ++nt)
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                const int c = 8 * nt + 2 * tq + e;
                const float dist = msq[nt][e] - 2.0f * acc[nt][2 * hh + e];
                if (c < C && dist < best) {
                  best = dist;
                  bi = c;
                }
              }
#pragma unroll
            for (int o = 1; o <= 2; o <<= 1) {
              const float ob = __shfl_xor_sync(0xffffffffu, best, o);
              const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
              if (ob < best || (ob == best && oi < bi)) {
                best = ob;
                bi = oi;
              }
            }
            const int r = 16 * rt + gq + 8 * hh;
            if (tq == 0) assign[r] = r < rc ? bi : -1;
          }
        };
        const int nrt = (rc + 15) / 16;  // row tiles holding rows of the group
        // four row tiles at a time, so that four independent product chains
        // are in flight (rows past rc are zero and get assignment -1)
        constexpr int kRt = 4;
        for (int rt0 = 0; rt0 < kChunkRows / 16; rt0 += kRt) {
          if (rt0 >= nrt) {
            if (lane < 16 * kRt / 2) reinterpret_cast<int2*>(assign + 16 * rt0)[lane] = make_int2(-1, -1);
            continue;
          }
          float acc[kRt][NTC][4];
#pragma unroll
          for (int t = 0; t < kRt; ++t)
#pragma unroll
            for (int i = 0; i < NTC; ++i)
#pragma unroll
              for (int k = 0; k < 4; ++k) acc[t][i][k] = 0.0f;
#pragma unroll
          for (int ks = 0; ks < KSTEPS; ++ks) {
            uint32_t a[kRt][4];
#pragma unroll
            for (int t = 0; t < kRt; ++t)
              ldsm_x4(a[t], xs_base + 2u * ((16 * (rt0 + t) + a_row) * XS + ks * 16 + a_col));
            // the hi and lo products of one accumulator are kRt * NTC issues apart
#pragma unroll
            for (int t = 0; t < kRt; ++t)
#pragma unroll
              for (int nt = 0; nt < NTC; ++nt) mma_16816(acc[t][nt], a[t], bhi[nt][ks][0], bhi[nt][ks][1]);
#pragma unroll
            for (int t = 0; t < kRt; ++t)
#pragma unroll
              for (int nt = 0; nt < NTC; ++nt) mma_16816(acc[t][nt], a[t], blo[nt][ks][0], blo[nt][ks][1]);
          }
#pragma unroll
          for (int t = 0; t < kRt; ++t) pick(rt0 + t, acc[t]);
        }
        __syncwarp();
        // cluster sums (and counts, from the column of ones): one-hot^T x
        for (int k0 = 0; k0 < rc; k0 += 16) {
          uint32_t a[4];
          const int ka = k0 + 2 * tq, kb = ka + 8;
          const int s0 = assign[ka], s1 = assign[ka + 1], s2 = assign[kb], s3 = assign[kb + 1];
          const uint32_t one = 0x3F80u;
          a[0] = (s0 == gq ? one : 0u) | ((s1 == gq ? one : 0u) << 16);
          a[1] = (s0 == gq + 8 ? one : 0u) | ((s1 == gq + 8 ? one : 0u) << 16);
          a[2] = (s2 == gq ? one : 0u) | ((s3 == gq ? one : 0u) << 16);
          a[3] = (s2 == gq + 8 ? one : 0u) | ((s3 == gq + 8 ? one : 0u) << 16);
#pragma unroll
          for (int p = 0; p < D / 16; ++p) {
            uint32_t b[4];
            ldsm_x4_trans(b, xs_base + 2u * ((k0 + t_row) * XS + 16 * p + t_col));
            mma_16816(sums[2 * p], a, b[0], b[1]);
            mma_16816(sums[2 * p + 1], a, b[2], b[3]);
          }
          uint32_t b2[2];
          ldsm_x2_trans(b2, xs_base + 2u * ((k0 + (lane & 15)) * XS + D));
          mma_16816(sums[D / 8], a, b2[0], b2[1]);
        }
      }
      // counts: column 0 of the last n-tile, held by the quad's first lane
#pragma unroll
      for (int h = 0; h < NTC; ++h)
        cnt[h] = static_cast<int>(__shfl_sync(0xffffffffu, sums[D / 8][2 * h], lane & ~3));
      // update: mu_c = sum_c / n_c in the registers the next round reads
#pragma unroll
      for (int h = 0; h < NTC; ++h) {
        const int c = gq + 8 * h;
        if (c < C && cnt[h] > 0) {
          const float inv = 1.0f / static_cast<float>(cnt[h]);
#pragma unroll
          for (int ks = 0; ks < KSTEPS; ++ks) {
            mu[h][ks][0] = sums[2 * ks][2 * h] * inv;
            mu[h][ks][1] = sums[2 * ks][2 * h + 1] * inv;
            mu[h][ks][2] = sums[2 * ks + 1][2 * h] * inv;
            mu[h][ks][3] = sums[2 * ks + 1][2 * h + 1] * inv;
          }
        }
      }
    }
    const int64_t t = bh * G + g;
#pragma unroll
    for (int h = 0; h < NTC; ++h) {
      const int c = gq + 8 * h;
      if (c < C) {
        float* dst = centroids + (t * C + c) * D;
#pragma unroll
        for (int ks = 0; ks < KSTEPS; ++ks) {
          *reinterpret_cast<float2*>(dst + 16 * ks + 2 * tq) = make_float2(mu[h][ks][0], mu[h][ks][1]);
          *reinterpret_cast<float2*>(dst + 16 * ks + 8 + 2 * tq) = make_float2(mu[h][ks][2], mu[h][ks][3]);
        }
        if (tq == 0) counts[t * C + c] = cnt[h];
      }
    }
  }
}


// --------------------------------------- k-means on tcgen05 (d = 128)
// Groups of at most 128 rows.  A persistent CTA per SM streams the groups'
// 128-row Q tiles through a ring of kKtSlots shared-memory buffers (TMA,
// 128-byte swizzle), and kKtSets sets of four warps each run one group's
// k-means at a time, every round on the tile in shared memory:
//   assign  S = X [hi | lo]^T (M = 128 rows, N = 2 C', K = d; the set writes
//           the centroids' bf16 hi and lo parts as an MN-major operand); one
//           thread per row (TMEM lane) takes argmin_c |mu_c|^2 - 2 (S_hi,c +
//           S_lo,c), ties to the lower c, and writes its row of the one-hot
//           matrix OH (MN-major: 128 rows x 16 cluster slots);
//   update  Sum^T = X^T OH (M = d dimensions, N = 16, K = 128 rows; the same
//           X tile read MN-major); one thread per dimension (TMEM lane)
//           multiplies its row of Sum^T by the reciprocal counts (ballots of
//           the labels); an empty cluster keeps its centroid.
// Thread t of a set keeps mu_c[t] for every c in registers across rounds.  A
// set issues its own MMAs (one elected lane of its first warp) and waits for
// them on its own barrier, so one set's waits overlap the other sets' work.
// The operands a set writes (centroid parts, one-hot rows) are 16-byte rows
// of the no-swizzle MN-major layout: 8 consecutive N entries of one K index
// per 16 bytes, so each thread stores whole vectors.
// Warp 4 kKtSets is the TMA producer.  Every wait is bounded.
// With C' = 8 the kernel also computes key means (FUSE): kKbWarps more warps
// stream K, which the k-means leaves most of HBM's bandwidth free for,
// through their own small cp.async rings in the shared memory the k-means
// does not use.  They take key blocks from a counter in global memory and
// stop taking more once the CTA's k-means sets are done; key_means_rest_kernel
// then takes the blocks left.  Both write kbar exactly as key_means_kernel
// does (the same lane-to-dimension map and the same order of the sums).
constexpr int kKtSets = 4;
constexpr int kKtSlots = 5;
constexpr int kKtThreads = (4 * kKtSets + 1) * 32;
constexpr int kKbWarps = 6;    // key-mean warps of the fused kernel
constexpr int kKbStages = 2;   // ring chunks per key-mean warp
constexpr int kKbRows = 8;     // key rows per chunk
constexpr uint32_t kKbChunk = kKbRows * 128 * 2;
constexpr int kKtThreadsFused = kKtThreads + kKbWarps * 32;

template <int CP>
struct KtLayout {
  static constexpr uint32_t kXBytes = 128 * 128 * 2;  // 128 rows x 128 dims, two 64-dim boxes
  static constexpr uint32_t kBox = 128 * 128;
  static constexpr uint32_t kX = 0;
  // MN-major no-swizzle operands: the 8-entry N group j of K index k at
  // j * kNGroup + k * 16 (K groups of 8 packed at 128-byte steps)
  static constexpr uint32_t kNGroup = 128 * 16;
  static constexpr uint32_t kMcBytes = (2 * CP / 8) * kNGroup;  // hi groups, then lo groups
  static constexpr uint32_t kOhBytes = 2 * kNGroup;             // 16 cluster slots
  static constexpr uint32_t kMc = kKtSlots * kXBytes;
  static constexpr uint32_t kOh = kMc + kKtSets * kMcBytes;
  // per set: |mu|^2 partials [16][4], |mu|^2 [16], counts [16], reciprocal
  // counts [16], count partials [16][4]
  static constexpr uint32_t kRed = kOh + kKtSets * kOhBytes;
  static constexpr uint32_t kRedBytes = (64 + 16 + 16 + 16 + 64) * 4;
  static constexpr uint32_t kBar = kRed + kKtSets * kRedBytes;
  static constexpr int kXFull = 0, kXEmpty = kKtSlots, kMmaDone = 2 * kKtSlots, kNumBars = 2 * kKtSlots + kKtSets;
  static constexpr uint32_t kMisc = kBar + kNumBars * 8;  // TMEM address, abort flag; released[] at +16
  static constexpr uint32_t kAlloc = kMisc + 16 + 4 * kKtSlots + 1024;
  // fused kernel: the count of k-means sets done, the key-mean warps' chunk
  // descriptors [kKbWarps][kKbStages] (block, offset << 8 | rows), their rings
  static constexpr uint32_t kKb = (kMisc + 16 + 4 * kKtSlots + 15) & ~15u;
  static constexpr uint32_t kKbDesc = kKb + 16;
  static constexpr uint32_t kKbRing = (kKbDesc + kKbWarps * kKbStages * 8 + 15) & ~15u;
  static constexpr uint32_t kAllocFused = kKbRing + kKbWarps * kKbStages * kKbChunk + 1024;
};

// Byte offset of element (row r, column c) in a K-major 128-byte-swizzled
// tile of `rows` rows whose columns come in 64-element chunks.
__device__ __forceinline__ uint32_t sw128_off(int rows, int r, int c) {
  return static_cast<uint32_t>((c >> 6) * rows * 128 + r * 128 + ((((c & 63) >> 3) ^ (r & 7)) << 4) + (c & 7) * 2);
}

// Sums v[0 .. CP) over the warp's lanes: lane l ends with the total of
// element e(l) = sum over the halving steps of (lane bit set) * (half size).
template <int CP>
__device__ __forceinline__ float warp_sum_scatter(float (&v)[CP], int lane, int& elem) {
  int base = 0;
#pragma unroll
  for (int half = CP / 2, o = 16; half >= 1; half >>= 1, o >>= 1) {
    const bool up = (lane & o) != 0;
#pragma unroll
    for (int j = 0; j < half; ++j) {
      const float send = up ? v[j] : v[j + half];
      const float keep = up ? v[j + half] : v[j];
      v[j] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
    base += up ? half : 0;
  }
  float r = v[0];
  // the lane bits the halving steps did not use
#pragma unroll
  for (int o = 32 / CP / 2; o >= 1; o >>= 1) r += __shfl_xor_sync(0xffffffffu, r, o);
  elem = base;
  return r;
}

template <int CP, bool FUSE>
__global__ void __launch_bounds__(FUSE ? kKtThreadsFused : kKtThreads, 1)
    kmeans_tc_kernel(const __grid_constant__ CUtensorMap tm_q, int BH, int N, int G, int q_block,
                     const int32_t* __restrict__ off, int C, int iters, float* __restrict__ centroids,
                     int32_t* __restrict__ counts, uint64_t timeout_ns, int* status,
                     const uint16_t* __restrict__ kmat, int Bk, int nK, uint16_t* __restrict__ kbar_hi,
                     uint16_t* __restrict__ kbar_lo, uint32_t* __restrict__ kb_next) {
  using namespace isa_dev;
  using L = KtLayout<CP>;
  constexpr int D = 128;
  constexpr int kProducer = 4 * kKtSets;
  constexpr int NG = CP / 8;  // 8-entry groups per centroid part
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  auto bar = [&](int i) -> uint32_t { return base + L::kBar + 8u * static_cast<uint32_t>(i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  // released[slot]: how many uses of the slot have been handed back
  volatile uint32_t* released = reinterpret_cast<volatile uint32_t*>(smem + L::kMisc + 16);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t n_items = static_cast<int64_t>(BH) * G;

  if (tid == 0) {
    for (int i = 0; i < kKtSlots; ++i) released[i] = 0u;
    for (int i = 0; i < kKtSlots; ++i) {
      mbar_init(bar(L::kXFull + i), 1);
      mbar_init(bar(L::kXEmpty + i), 1);
    }
    for (int i = 0; i < kKtSets; ++i) mbar_init(bar(L::kMmaDone + i), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  // one-hot slots of clusters >= C stay zero, and the counts start at zero
  if constexpr (FUSE) {
    if (tid == 0) *reinterpret_cast<volatile int*>(smem + L::kKb) = 0;
  }
  if (tid < kKtThreads) {
    for (int i = tid; i < static_cast<int>(kKtSets * L::kOhBytes / 16); i += kKtThreads)
      reinterpret_cast<uint4*>(smem + L::kOh)[i] = make_uint4(0u, 0u, 0u, 0u);
    for (int i = tid; i < static_cast<int>(kKtSets * L::kRedBytes / 4); i += kKtThreads)
      reinterpret_cast<uint32_t*>(smem + L::kRed)[i] = 0u;
  }
  fence_proxy_async_smem();
  if (warp == kProducer) {
    tmem_alloc(smem_addr(tmem_slot), 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // rows [r0, r0 + n) of group `item`; n = 0 for malformed offsets
  auto rows_of = [&](int64_t item, int64_t& bh, int& g, int& r0, int& n, bool& malformed) {
    bh = item / G;
    g = static_cast<int>(item - bh * G);
    malformed = false;
    if (off) {
      r0 = off[g];
      const int r1 = off[g + 1];
      if (r0 < 0 || r1 > N || r1 <= r0) {
        malformed = true;
        r0 = 0;
        n = 0;
      } else {
        n = r1 - r0;
      }
    } else {
      r0 = g * q_block;
      n = min(N, r0 + q_block) - r0;
    }
  };

  if (warp == kProducer) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      uint32_t k = 0, loads = 0;
      for (int64_t item = blockIdx.x; item < n_items; item += gridDim.x, ++k) {
        const uint32_t slot = k % kKtSlots, use = k / kKtSlots;
        if (!mbar_wait(bar(L::kXEmpty + slot), (use & 1u) ^ 1u, abort_flag, timeout_ns)) break;
        int64_t bh;
        int g, r0, n;
        bool bad;
        rows_of(item, bh, g, r0, n, bad);
        if (n >= 1 && n <= 128) {
          mbar_arrive_expect_tx(bar(L::kXFull + slot), L::kXBytes);
#pragma unroll
          for (int c = 0; c < D / 64; ++c)
            tma_load_3d(base + L::kX + slot * L::kXBytes + c * L::kBox, &tm_q, bar(L::kXFull + slot), c * 64, r0,
                        static_cast<int32_t>(bh));
        } else {
          mbar_arrive(bar(L::kXFull + slot));  // nothing to load for this group
        }
        loads = k + 1;
      }
      if (*abort_flag) {
        // let the copies already issued land before the CTA leaves
        const uint32_t first = loads > kKtSlots ? loads - kKtSlots : 0;
        for (uint32_t i = first; i < loads; ++i) {
          const uint64_t t0 = global_timer_ns();
          while (!mbar_try_wait(bar(L::kXFull + i % kKtSlots), (i / kKtSlots) & 1u))
            if (global_timer_ns() - t0 > 200000000ull) break;
        }
      }
    }
  } else if (warp < kProducer) {
    // ------------------------------------------------------- k-means sets
    const int s = warp >> 2, q4 = warp & 3;
    const int t = q4 * 32 + lane;  // TMEM lane: the X row (assign) or the dimension (update)
    // the set's MMA-issuing warp sits on SM sub-partition s, so that no two
    // issuing warps share one; the next warp finishes the norms and counts
    const int q_mma = s & 3, q_aux = (s + 1) & 3;
    const uint32_t bar_id = 1u + static_cast<uint32_t>(s);
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const uint32_t col_s = 64u * s, col_u = 64u * s + 32u;
    const uint32_t mc = base + L::kMc + s * L::kMcBytes;
    const uint32_t oh = base + L::kOh + s * L::kOhBytes;
    uint4* mc_row = reinterpret_cast<uint4*>(smem + L::kMc + s * L::kMcBytes) + t;  // K index t of N group 0
    uint4* oh_row = reinterpret_cast<uint4*>(smem + L::kOh + s * L::kOhBytes) + t;
    float* nsq_part = reinterpret_cast<float*>(smem + L::kRed + s * L::kRedBytes);  // [16][4]
    float* nsq_fin = nsq_part + 64;                                                // [16]
    uint32_t* cnt = reinterpret_cast<uint32_t*>(nsq_fin + 16);                      // [16]
    float* inv = reinterpret_cast<float*>(cnt + 16);                               // [16]
    uint32_t* cnt_part = reinterpret_cast<uint32_t*>(inv + 16);                    // [16][4]
    constexpr uint32_t idesc_assign = idesc_bf16_f32(128, 2 * CP, 1, 0);
    constexpr uint32_t idesc_update = idesc_bf16_f32(128, 16, 1, 1);
    uint32_t mma_waits = 0;
    bool pending = false;  // an MMA batch was committed and not yet waited for
    bool ok = true;
    // waits for this set's last MMA batch; the set agrees on the outcome
    auto wait_mma = [&]() -> bool {
      bool good = true;
      if (q4 == q_mma) good = mbar_wait_warp(bar(L::kMmaDone + s), mma_waits & 1u, abort_flag, timeout_ns);
      good = named_bar_and(bar_id, 128, good);
      if (good) {
        ++mma_waits;
        pending = false;
        tc_fence_after();
      }
      return good;
    };
    // The sets take the slots' uses out of order (a set may be through with
    // a group before the group of the slot's previous use has even landed),
    // so before waiting on a slot's full barrier for use u a set waits until
    // uses 0 .. u-1 have been handed back: the barrier is then at most one
    // phase ahead of u and its parity cannot alias.
    auto wait_released = [&](uint32_t slot, uint32_t use) -> bool {
      const uint64_t t0 = global_timer_ns();
      uint32_t spins = 0;
      while (released[slot] != use) {
        if ((++spins & 63u) == 0) {
          if (*abort_flag) return false;
          if (global_timer_ns() - t0 > timeout_ns) {
            *abort_flag = 1;
            return false;
          }
        }
      }
      return true;
    };
    // hands a slot back to the producer (thread 0 of the set)
    auto release_slot = [&](uint32_t slot, uint32_t use) {
      if (t == 0) {
        released[slot] = use + 1u;
        __threadfence_block();
        mbar_arrive(bar(L::kXEmpty + slot));
      }
    };
    uint32_t k = static_cast<uint32_t>(s);
    for (int64_t item = blockIdx.x + static_cast<int64_t>(s) * gridDim.x; item < n_items && ok;
         item += static_cast<int64_t>(kKtSets) * gridDim.x, k += kKtSets) {
      const uint32_t slot = k % kKtSlots, use = k / kKtSlots;
      int64_t bh;
      int g, r0, n;
      bool bad;
      rows_of(item, bh, g, r0, n, bad);
      bool got = true;
      if (q4 == 0) {
        got = __all_sync(0xffffffffu, wait_released(slot, use));
        if (got) got = mbar_wait_warp(bar(L::kXFull + slot), use & 1u, abort_flag, timeout_ns);
      }
      got = named_bar_and(bar_id, 128, got);
      if (!got) {
        ok = false;
        break;
      }
      if (n > 128) {  // a larger group: the warp-per-group kernel runs it
        release_slot(slot, use);
        continue;
      }
      if (bad && t == 0) atomicCAS(status, 0, kStatusDeviceCheck);
      const uint32_t xs = base + L::kX + slot * L::kXBytes;
      const uint8_t* xp = smem + L::kX + slot * L::kXBytes;
      // thread t's dimension of every centroid, initialised at rows floor(c n / C)
      float mu[CP];
#pragma unroll
      for (int c = 0; c < CP; ++c) {
        const int r = (c < C && n > 0) ? static_cast<int>((static_cast<int64_t>(c) * n) / C) : -1;
        mu[c] = r < 0 ? 0.0f : bf16_to_f(*reinterpret_cast<const uint16_t*>(xp + sw128_off(128, r, t)));
      }
      uint32_t my_count = 0;  // the count of cluster t (t < C) from the last assignment
      for (int it = 0; it < iters && n > 0; ++it) {
        // ---- centroid operands (hi and lo parts, MN-major) and |mu_c|^2 partials
        {
          uint32_t hi[CP / 2], lo[CP / 2];
          float p[CP];
#pragma unroll
          for (int j = 0; j < CP / 2; ++j) {
            hi[j] = pack_bf16x2(mu[2 * j], mu[2 * j + 1]);
            lo[j] = pack_bf16x2(mu[2 * j] - __uint_as_float(hi[j] << 16),
                                mu[2 * j + 1] - __uint_as_float(hi[j] & 0xFFFF0000u));
          }
#pragma unroll
          for (int j = 0; j < NG; ++j) {
            mc_row[j * (L::kNGroup / 16)] = make_uint4(hi[4 * j], hi[4 * j + 1], hi[4 * j + 2], hi[4 * j + 3]);
            mc_row[(NG + j) * (L::kNGroup / 16)] = make_uint4(lo[4 * j], lo[4 * j + 1], lo[4 * j + 2], lo[4 * j + 3]);
          }
#pragma unroll
          for (int c = 0; c < CP; ++c) p[c] = mu[c] * mu[c];
          int e;
          const float ps = warp_sum_scatter<CP>(p, lane, e);
          if ((lane & (32 / CP - 1)) == 0) nsq_part[e * 4 + q4] = ps;
        }
        fence_proxy_async_smem();
        tc_fence_before();
        named_bar_sync(bar_id, 128);
        // ---- S = X [hi | lo]^T, while warp 1 finishes the norms and clears the counts
        if (q4 == q_mma) {
          tc_fence_after();
          const uint64_t da = smem_desc_sw128(xs, 16, 1024), db = smem_desc_none(mc, 128, L::kNGroup);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t oa = ((kk >> 2) * L::kBox + (kk & 3) * 32) >> 4;
            if (elect_one()) mma_ss(tmem + col_s, da + oa, db + ((kk * 256) >> 4), idesc_assign, kk > 0 ? 1u : 0u);
          }
          if (elect_one()) tc_commit(bar(L::kMmaDone + s));
        } else if (q4 == q_aux && lane < CP) {
          const float4 np = *reinterpret_cast<const float4*>(nsq_part + 4 * lane);
          nsq_fin[lane] = (np.x + np.y) + (np.z + np.w);
        }
        pending = true;
        if (!wait_mma()) {
          ok = false;
          break;
        }
        // ---- assignment: thread t = row t of the tile
        int label = -1;
        {
          uint32_t sv[16];
          tmem_ld16(lane_base + col_s, sv);
          uint32_t sv2[16];
          if constexpr (CP == 16) tmem_ld16(lane_base + col_s + 16, sv2);
          tmem_wait_ld();
          float nsq[CP];
#pragma unroll
          for (int j = 0; j < CP / 4; ++j) {
            const float4 v4 = reinterpret_cast<const float4*>(nsq_fin)[j];
            nsq[4 * j] = v4.x;
            nsq[4 * j + 1] = v4.y;
            nsq[4 * j + 2] = v4.z;
            nsq[4 * j + 3] = v4.w;
          }
          float best = INFINITY;
          int bi = 0;
#pragma unroll
          for (int c = 0; c < CP; ++c) {
            const uint32_t s_hi = CP == 16 ? (c < 16 ? sv[c] : 0u) : sv[c];
            const uint32_t s_lo = CP == 16 ? sv2[c] : sv[CP + c];
            const float dot = __uint_as_float(s_hi) + __uint_as_float(s_lo);
            const float dist = nsq[c] - 2.0f * dot;
            if (c < C && dist < best) {
              best = dist;
              bi = c;
            }
          }
          label = t < n ? bi : -1;
        }
        // one-hot row t: slot `label` holds 1.0 (bf16 0x3F80)
        {
          const uint32_t w1 = 0x3F80u << ((label & 1) << 4);
#pragma unroll
          for (int j = 0; j < NG; ++j) {
            uint32_t wd[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) wd[i] = (label >> 1) == 4 * j + i ? w1 : 0u;
            oh_row[j * (L::kNGroup / 16)] = make_uint4(wd[0], wd[1], wd[2], wd[3]);
          }
        }
        // this warp's count of each cluster: one ballot per cluster
#pragma unroll
        for (int c = 0; c < CP; ++c) {
          if (c < C) {
            const uint32_t b = __ballot_sync(0xffffffffu, label == c);
            if (lane == 0) cnt_part[c * 4 + q4] = static_cast<uint32_t>(__popc(b));
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        named_bar_sync(bar_id, 128);
        // ---- Sum^T = X^T OH, while warp 1 takes the reciprocal counts
        if (q4 == q_mma) {
          tc_fence_after();
          const uint64_t da = smem_desc_sw128(xs, L::kBox, 1024), db = smem_desc_none(oh, 128, L::kNGroup);
#pragma unroll
          for (int kk = 0; kk < 128 / 16; ++kk)
            if (elect_one())
              mma_ss(tmem + col_u, da + ((kk * 2048) >> 4), db + ((kk * 256) >> 4), idesc_update, kk > 0 ? 1u : 0u);
          if (elect_one()) tc_commit(bar(L::kMmaDone + s));
        } else if (q4 == q_aux && lane < CP) {
          const uint4 cp4 = *reinterpret_cast<const uint4*>(cnt_part + 4 * lane);
          const uint32_t cc = lane < C ? (cp4.x + cp4.y) + (cp4.z + cp4.w) : 0u;
          cnt[lane] = cc;
          inv[lane] = cc > 0u ? 1.0f / static_cast<float>(cc) : 0.0f;
        }
        pending = true;
        if (!wait_mma()) {
          ok = false;
          break;
        }
        if (it == iters - 1) release_slot(slot, use);  // X is no longer read
        // ---- update: thread t = dimension t
        {
          uint32_t uv[16];
          tmem_ld16(lane_base + col_u, uv);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < CP / 4; ++j) {
            const float4 i4 = reinterpret_cast<const float4*>(inv)[j];
            const float iv[4] = {i4.x, i4.y, i4.z, i4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int c = 4 * j + e;
              if (iv[e] > 0.0f) mu[c] = __uint_as_float(uv[c]) * iv[e];
            }
          }
          if (t < C) my_count = cnt[t];
        }
      }
      if (!ok) break;
      if (n == 0) release_slot(slot, use);
      const int64_t o = bh * G + g;
#pragma unroll
      for (int c = 0; c < CP; ++c)
        if (c < C) centroids[(o * C + c) * D + t] = mu[c];
      if (t < C) counts[o * C + t] = static_cast<int32_t>(my_count);
    }
    if constexpr (FUSE) {
      // this set takes no more groups: the key-mean warps stop taking blocks
      // once every set of the CTA is here
      __syncwarp();
      if (q4 == 0 && lane == 0) atomicAdd(reinterpret_cast<int*>(smem + L::kKb), 1);
    }
    if (pending && q4 == q_mma) {
      // a batch whose wait gave up may still be running: let it finish before
      // the tensor memory is freed
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(bar(L::kMmaDone + s), mma_waits & 1u))
        if (global_timer_ns() - t0 > 200000000ull) break;
    }
  } else if constexpr (FUSE) {
    // ------------------------------------------------- key means (fused)
    // The warp takes kb_run key blocks at a time from *kb_next and streams
    // their rows through its ring in chunks of at most kKbRows rows, a chunk
    // never crossing a block (each lane copies up to four 16-byte pieces);
    // the chunk's (block, offset, rows) goes to the warp's descriptor slot.
    // Lane l sums dimensions 4l .. 4l + 3 of every row in order, and the
    // block's last chunk writes its mean.  No block is taken once all of the
    // CTA's k-means sets are done; the stream then ends with the chunks in
    // flight.
    const int kw = warp - kProducer - 1;
    const int n_blk = BH * nK;
    const int kb_run = Bk >= 64 ? 1 : 64 / Bk;
    volatile int* sets_done = reinterpret_cast<volatile int*>(smem + L::kKb);
    volatile int* desc = reinterpret_cast<volatile int*>(smem + L::kKbDesc) + 2 * kw * kKbStages;
    const uint32_t ring = base + L::kKbRing + static_cast<uint32_t>(kw) * (kKbStages * kKbChunk);
    const uint8_t* ring_p = smem + L::kKbRing + static_cast<uint32_t>(kw) * (kKbStages * kKbChunk);
    auto rows_of_block = [&](int b) -> int {
      const int kb = b % nK;
      return min(N, (kb + 1) * Bk) - kb * Bk;
    };
    // issue side (warp-uniform): the block being cut into chunks, the end of
    // the run it belongs to, the next chunk's row offset in it
    int cur_b = 0, run_end = 0, cur_off = 0;
    bool more = true;
    auto issue = [&](int c) {
      int b = -1, o = 0, rows = 0;
      if (more && cur_b >= run_end) {
        int r0 = n_blk;
        if (lane == 0 && *sets_done < kKtSets) r0 = static_cast<int>(atomicAdd(kb_next, static_cast<uint32_t>(kb_run)));
        r0 = __shfl_sync(0xffffffffu, r0, 0);
        if (r0 >= n_blk) {
          more = false;
        } else {
          cur_b = r0;
          run_end = min(n_blk, r0 + kb_run);
          cur_off = 0;
        }
      }
      if (more) {
        b = cur_b;
        o = cur_off;
        const int rb = rows_of_block(b);
        rows = min(kKbRows, rb - o);
        cur_off += rows;
        if (cur_off >= rb) {
          ++cur_b;
          cur_off = 0;
        }
        const int bh = b / nK, kb = b - bh * nK;
        const uint16_t* src = kmat + (static_cast<int64_t>(bh) * N + static_cast<int64_t>(kb) * Bk + o) * 128;
        const uint32_t dst = ring + static_cast<uint32_t>(c % kKbStages) * kKbChunk;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int piece = lane + 32 * j;  // 16-byte piece of the chunk; row piece / 16
          if ((piece >> 4) < rows) cp_async16(dst + piece * 16, src + piece * 8);
        }
      }
      if (lane == 0) {
        desc[2 * (c % kKbStages)] = b;
        desc[2 * (c % kKbStages) + 1] = (o << 8) | rows;
      }
      cp_async_commit();  // an empty group past the end keeps the count regular
    };
#pragma unroll
    for (int c = 0; c < kKbStages - 1; ++c) issue(c);
    float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    for (int c = 0;; ++c) {
      issue(c + kKbStages - 1);
      cp_async_wait_group<kKbStages - 1>();  // this lane's pieces of chunk c have landed
      __syncwarp();                           // and the other lanes' too, and its descriptor
      const int d_b = desc[2 * (c % kKbStages)], d_or = desc[2 * (c % kKbStages) + 1];
      if (d_b < 0) break;
      const int rows = d_or & 255, o = d_or >> 8;
      const uint8_t* chunk = ring_p + static_cast<uint32_t>(c % kKbStages) * kKbChunk;
      for (int i = 0; i < rows; ++i) {
        const uint2 v = *reinterpret_cast<const uint2*>(chunk + i * 256 + lane * 8);
        acc[0] += bf16_to_f(v.x & 0xFFFF);
        acc[1] += bf16_to_f(v.x >> 16);
        acc[2] += bf16_to_f(v.y & 0xFFFF);
        acc[3] += bf16_to_f(v.y >> 16);
      }
      const int rb = rows_of_block(d_b);
      if (o + rows == rb) {
        const float inv = 1.0f / static_cast<float>(rb);
        const int64_t out = static_cast<int64_t>(d_b) * 128 + lane * 4;  // (bh nK + b) d
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float m = acc[e] * inv;
          const uint16_t hi = bf16_bits_rn(m);
          kbar_hi[out + e] = hi;
          kbar_lo[out + e] = bf16_bits_rn(m - bf16_bits_to_f(hi));
          acc[e] = 0.0f;
        }
      }
      __syncwarp();  // every lane has read the chunk and its descriptor before the slot is reused
    }
    cp_async_wait_group<0>();
  }
  tc_fence_before();
  __syncthreads();
  if (tid == 0 && *abort_flag) atomicCAS(status, 0, kStatusTimeout);
  if (warp == kProducer) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// ------------------------------------------------------------------ mass
// One CTA per (batch*head, 128 centroid rows = 128 / Cp groups; Cp = C
// rounded up to a power of two, padding rows carry weight 0).
//   logits  l_{c,b} = scale mu_c . kbar_b (+ ln(L_b / Bk) on a partial tail
//           block; the common ln Bk cancels in the softmax), computed on
//           tensor cores: mu and kbar are bf16 hi + lo pairs and three
//           tcgen05.mma products (hi.hi + hi.lo + lo.hi) accumulate in TMEM;
//   pass 0  each row's online max and sum of exp over all key blocks;
//   pass 1  the logits again, p = n_c exp(l - max) / sum, summed over the Cp
//           rows of each group through a shared-memory transpose, and written.
// Warps 0-7: softmax, two warps per centroid row quarter (TMEM lanes
// 32 (w & 3) ..), warp w taking columns 64 (w >> 2) .. + 63 of every tile;
// warp 8: TMA producer of the kbar tiles (128 blocks x d, hi and lo) into a
// 2-stage ring; warp 9: MMA issue.  S is double-buffered in TMEM (2 x 128
// columns).
constexpr int kMassSoftmaxWarps = 8;
constexpr int kMassThreads = (kMassSoftmaxWarps + 2) * 32;
constexpr int kMassRing = 2;

template <int D>
struct MassLayout {
  static constexpr uint32_t kTile = 128 * D * 2;           // one 128-row bf16 tile
  static constexpr uint32_t kChunk = 128 * 128;            // 128 rows x 64 bf16
  static constexpr uint32_t kAHi = 0, kALo = kTile, kRing = 2 * kTile;
  static constexpr uint32_t kStage = 2 * kTile;            // kbar hi + lo
  static constexpr uint32_t kBar = kRing + kMassRing * kStage;
  static constexpr int kBarFull = 0, kBarEmpty = kMassRing, kBarSFull = 2 * kMassRing, kBarSFree = kBarSFull + 2,
                       kBarFinal = kBarSFree + 2, kBarXchg = kBarFinal + 1, kNumBars = kBarXchg + 1;
  static constexpr uint32_t kMisc = kBar + kNumBars * 8;
  static constexpr uint32_t kXchg = (kMisc + 16 + 15) & ~15u;  // [2 halves][128 rows] (max, sum)
  static constexpr int kXS = 20;  // row stride (floats) of the transpose buffers: 16 columns + 4
  static constexpr uint32_t kXpose = kXchg + 2 * 128 * 8;
  static constexpr uint32_t kAlloc = kXpose + kMassSoftmaxWarps * 32 * kXS * 4 + 1024;
};

template <int D, int Cp>
__global__ void __launch_bounds__(kMassThreads, 1)
    mass_kernel(const __grid_constant__ CUtensorMap tm_hi, const __grid_constant__ CUtensorMap tm_lo,
                const float* __restrict__ centroids, const int32_t* __restrict__ counts, int N, int Bk, int nK,
                int G, int C, float scale_log2, float* __restrict__ mass, int* status) {
  using namespace isa_dev;
  using L = MassLayout<D>;
  constexpr int kGroupsPerTile = 128 / Cp;
  constexpr int kProducer = kMassSoftmaxWarps, kMma = kMassSoftmaxWarps + 1;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  auto bar = [&](int i) -> uint32_t { return base + L::kBar + 8u * static_cast<uint32_t>(i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t bh = blockIdx.y;
  const int g0 = blockIdx.x * kGroupsPerTile;
  const int T = (nK + 127) / 128;
  const int n_items = 2 * T;

  // The producer thread sets up the barriers and starts the first k-bar tiles
  // on their way before the centroid conversion below: they do not depend on
  // it, and the other threads touch no barrier before the block-wide sync.
  auto load_item = [&](int i) {
    const uint32_t slot = i % kMassRing;
    mbar_arrive_expect_tx(bar(L::kBarFull + slot), L::kStage);
    const uint32_t dst = base + L::kRing + slot * L::kStage;
    const int row = (i % T) * 128;
#pragma unroll
    for (int c = 0; c < D / 64; ++c) {
      tma_load_3d(dst + c * L::kChunk, &tm_hi, bar(L::kBarFull + slot), c * 64, row, static_cast<int>(bh));
      tma_load_3d(dst + L::kTile + c * L::kChunk, &tm_lo, bar(L::kBarFull + slot), c * 64, row,
                  static_cast<int>(bh));
    }
  };
  const int pre = n_items < kMassRing ? n_items : kMassRing;  // loads issued before the sync
  if (warp == kProducer && lane == 0) {
    for (int i = 0; i < kMassRing; ++i) {
      mbar_init(bar(L::kBarFull + i), 1);
      mbar_init(bar(L::kBarEmpty + i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(L::kBarSFull + i), 1);
      mbar_init(bar(L::kBarSFree + i), kMassSoftmaxWarps * 32);
    }
    mbar_init(bar(L::kBarFinal), 1);
    mbar_init(bar(L::kBarXchg), kMassSoftmaxWarps * 32);
    *abort_flag = 0;
    fence_mbar_init();
    for (int i = 0; i < pre; ++i) load_item(i);
  }
  // centroid rows -> bf16 hi / lo, K-major with the 128-byte swizzle (16-byte
  // granule q of row r stored at granule q ^ (r & 7) of the row).  Each thread
  // issues the loads of all its granules before it converts any, so that
  // the global-memory latency is paid once.
  constexpr int kPer = (128 * (D / 8) + kMassThreads - 1) / kMassThreads;
  float4 ld[kPer][2];
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    const int i = tid + u * kMassThreads;
    const int r = i / (D / 8), q = i - r * (D / 8);
    const int gl = r / Cp, c = r - gl * Cp, g = g0 + gl;
    if (i < 128 * (D / 8) && c < C && g < G) {
      const float4* src = reinterpret_cast<const float4*>(centroids + ((bh * G + g) * C + c) * D + q * 8);
      ld[u][0] = src[0];
      ld[u][1] = src[1];
    } else {
      ld[u][0] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      ld[u][1] = ld[u][0];
    }
  }
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    const int i = tid + u * kMassThreads;
    if (i >= 128 * (D / 8)) break;
    const int r = i / (D / 8), q = i - r * (D / 8);
    const float v[8] = {ld[u][0].x, ld[u][0].y, ld[u][0].z, ld[u][0].w,
                        ld[u][1].x, ld[u][1].y, ld[u][1].z, ld[u][1].w};
    uint32_t hi[4], lo[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint16_t h0 = bf16_bits_rn(v[2 * e]), h1 = bf16_bits_rn(v[2 * e + 1]);
      const uint16_t l0 = bf16_bits_rn(v[2 * e] - bf16_bits_to_f(h0));
      const uint16_t l1 = bf16_bits_rn(v[2 * e + 1] - bf16_bits_to_f(h1));
      hi[e] = static_cast<uint32_t>(h0) | (static_cast<uint32_t>(h1) << 16);
      lo[e] = static_cast<uint32_t>(l0) | (static_cast<uint32_t>(l1) << 16);
    }
    const int chunk = q >> 3, qq = q & 7;
    const uint32_t off = chunk * L::kChunk + r * 128 + ((qq ^ (r & 7)) << 4);
    *reinterpret_cast<uint4*>(smem + L::kAHi + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    *reinterpret_cast<uint4*>(smem + L::kALo + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
  }
  if (warp == kMma) {
    tmem_alloc(smem_addr(tmem_slot), 256);
    tmem_relinquish();
  }
  // the generic-proxy stores of the A tiles must be visible to the tensor cores
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kProducer) {
    // ------------------------------------------------------------ producer
    uint32_t issued = static_cast<uint32_t>(pre);
    bool ok = true;
    if (lane == 0) {
      for (int i = pre; i < n_items && ok; ++i) {
        const uint32_t slot = i % kMassRing, use = i / kMassRing;
        if (!mbar_wait(bar(L::kBarEmpty + slot), (use & 1u) ^ 1u, abort_flag, kWaitTimeoutNs)) {
          ok = false;
          break;
        }
        load_item(i);
        ++issued;
      }
      if (!ok || *abort_flag) {
        const uint32_t first = issued > kMassRing ? issued - kMassRing : 0;
        for (uint32_t i = first; i < issued; ++i) {
          const uint64_t t0 = global_timer_ns();
          while (!mbar_try_wait(bar(L::kBarFull + i % kMassRing), (i / kMassRing) & 1u))
            if (global_timer_ns() - t0 > 200000000ull) break;
        }
      }
    }
  } else if (warp == kMma) {
    // ----------------------------------------------------------------- MMA
    // The whole warp runs the loop and waits; one elected lane issues.  The
    // shared-memory descriptors are built once and advanced by adds to their
    // start-address field (addresses stay below 2^18: no carry out of it).
    {
      constexpr uint32_t idesc = idesc_bf16_f32(128, 128, 0);
      const uint64_t da_hi = smem_desc_sw128(base + L::kAHi, 16, 1024);
      const uint64_t da_lo = smem_desc_sw128(base + L::kALo, 16, 1024);
      const uint64_t db = smem_desc_sw128(base + L::kRing, 16, 1024);
      for (int i = 0; i < n_items; ++i) {
        const uint32_t slot = i % kMassRing, buf = i & 1;
        if (!mbar_wait_warp(bar(L::kBarFull + slot), (i / kMassRing) & 1u, abort_flag, kWaitTimeoutNs)) break;
        if (!mbar_wait_warp(bar(L::kBarSFree + buf), ((i >> 1) & 1u) ^ 1u, abort_flag, kWaitTimeoutNs)) break;
        tc_fence_after();
        const uint64_t b_hi = db + ((slot * L::kStage) >> 4), b_lo = b_hi + (L::kTile >> 4);
        const uint32_t d = tmem + buf * 128;
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint64_t off = ((k >> 2) * L::kChunk + (k & 3) * 32) >> 4;
          if (elect_one()) mma_ss(d, da_hi + off, b_hi + off, idesc, k > 0 ? 1u : 0u);
          if (elect_one()) mma_ss(d, da_hi + off, b_lo + off, idesc, 1u);
          if (elect_one()) mma_ss(d, da_lo + off, b_hi + off, idesc, 1u);
        }
        if (elect_one()) {
          tc_commit(bar(L::kBarEmpty + slot));
          tc_commit(bar(L::kBarSFull + buf));
        }
      }
      if (elect_one()) tc_commit(bar(L::kBarFinal));
      __syncwarp();
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(bar(L::kBarFinal), 0))
        if (global_timer_ns() - t0 > 200000000ull) break;
    }
  } else {
    // ------------------------------------------------------------- softmax
    // Thread = centroid row = TMEM lane; the two warps of a row quarter take
    // the two 64-column halves of every tile.  With s = scale log2(e) > 0
    // the log2-domain logit of block b is z_b = s x_b for the raw product
    // x_b (a partial tail block adds log2(L_b / Bk) to it, folded into x as
    // an offset; columns past nK become -inf), so the running max is taken
    // on x.  A half tile comes out of TMEM in one go and the S buffer is
    // released before any arithmetic.
    //   pass 0  m = max z and Z = sum 2^(z - m), online over the tiles; the
    //           two halves' (m, Z) are merged once through shared memory;
    //   pass 1  n_c 2^(z - m) / Z = 2^(s x - o) with o = m - log2(n_c / Z):
    //           one paired FMA and one ex2 per value; the Cp rows of each
    //           group are summed through a per-warp shared-memory transpose
    //           of 16 columns at a time (row stride 20 floats: the row
    //           writes are free of bank conflicts).
    const int quarter = warp & 3, half = warp >> 2;
    const int row = quarter * 32 + lane;  // centroid row == TMEM lane
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + half * 64;
    const int gl = row / Cp, c = row - gl * Cp, g = g0 + gl;
    const float n_c = (c < C && g < G) ? static_cast<float>(counts[(bh * G + g) * C + c]) : 0.0f;
    const int tail_rows = N - (nK - 1) * Bk;
    const float tail_dx =
        tail_rows < Bk ? log2f(static_cast<float>(tail_rows) / static_cast<float>(Bk)) / scale_log2 : 0.0f;
    constexpr int kCols = 16 / Cp > 0 ? 16 / Cp : 1;  // columns a lane sums and stores per 16-column chunk
    float* xp = reinterpret_cast<float*>(smem + L::kXpose) + warp * 32 * L::kXS;
    float2* xchg = reinterpret_cast<float2*>(smem + L::kXchg);
    const int p = lane & (Cp - 1), gw = lane / Cp;  // this lane's slice and group within the warp
    const uint64_t ss = f2_pack(scale_log2, scale_log2);
    float m_run = -INFINITY, z_run = 0.0f, o = INFINITY;
    for (int i = 0; i < n_items; ++i) {
      const int pass = i / T, j = i - pass * T;
      const uint32_t buf = i & 1;
      if (!mbar_wait(bar(L::kBarSFull + buf), (i >> 1) & 1u, abort_flag, kWaitTimeoutNs)) break;
      tc_fence_after();
      uint32_t sv[2][32];
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) tmem_ld32(lane_base + buf * 128 + 32 * cc, sv[cc]);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(bar(L::kBarSFree + buf));
      const int col0 = j * 128 + half * 64;
      if (j == T - 1) {
#pragma unroll
        for (int cc = 0; cc < 2; ++cc)
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int b = col0 + 32 * cc + e;
            float xv = __uint_as_float(sv[cc][e]);
            if (b == nK - 1) xv += tail_dx;
            sv[cc][e] = __float_as_uint(b < nK ? xv : -INFINITY);
          }
      }
      if (pass == 0) {
        float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int cc = 0; cc < 2; ++cc)
#pragma unroll
          for (int e = 0; e < 32; e += 8)
#pragma unroll
            for (int k = 0; k < 4; ++k)
              mx[k] = fmax3f(mx[k], __uint_as_float(sv[cc][e + k]), __uint_as_float(sv[cc][e + 4 + k]));
        const float xm = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
        const float m_new = fmaxf(m_run, xm * scale_log2);
        // a half tile past nK is all -inf: nothing to add
        if (m_new != -INFINITY) {
          const uint64_t nm = f2_pack(-m_new, -m_new);
          uint64_t part[4] = {0ull, 0ull, 0ull, 0ull};  // +0.0f pairs
#pragma unroll
          for (int cc = 0; cc < 2; ++cc)
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              float y0, y1;
              f2_unpack(fma_f32x2(f2_pack(__uint_as_float(sv[cc][e]), __uint_as_float(sv[cc][e + 1])), ss, nm), y0,
                        y1);
              part[(e >> 1) & 3] = add_f32x2(part[(e >> 1) & 3], f2_pack(fast_exp2(y0), fast_exp2(y1)));
            }
          const uint64_t p01 = add_f32x2(add_f32x2(part[0], part[1]), add_f32x2(part[2], part[3]));
          float s0, s1;
          f2_unpack(p01, s0, s1);
          z_run = (m_run == -INFINITY ? 0.0f : z_run * fast_exp2(m_run - m_new)) + (s0 + s1);
          m_run = m_new;
        }
        if (j == T - 1) {
          // merge the two halves' (m, Z) in a fixed order, so that both warps
          // of the row get the same o
          xchg[half * 128 + row] = make_float2(m_run, z_run);
          mbar_arrive(bar(L::kBarXchg));
          if (!mbar_wait(bar(L::kBarXchg), 0, abort_flag, kWaitTimeoutNs)) break;
          const float2 h0 = xchg[row], h1 = xchg[128 + row];
          const float m = fmaxf(h0.x, h1.x);
          const float z = (h0.x == -INFINITY ? 0.0f : h0.y * fast_exp2(h0.x - m)) +
                          (h1.x == -INFINITY ? 0.0f : h1.y * fast_exp2(h1.x - m));
          const float w = z > 0.0f ? n_c / z : 0.0f;
          o = w > 0.0f ? m - log2f(w) : INFINITY;
        }
      } else {
        const uint64_t no = f2_pack(-o, -o);
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          const int cc = ch >> 1, e0 = (ch & 1) * 16;
          float v[16];
#pragma unroll
          for (int e = 0; e < 16; e += 2) {
            float y0, y1;
            f2_unpack(fma_f32x2(f2_pack(__uint_as_float(sv[cc][e0 + e]), __uint_as_float(sv[cc][e0 + e + 1])), ss,
                                no),
                      y0, y1);
            v[e] = fast_exp2(y0);
            v[e + 1] = fast_exp2(y1);
          }
          __syncwarp();  // every lane has read the previous chunk
#pragma unroll
          for (int k = 0; k < 4; ++k)
            *reinterpret_cast<float4*>(xp + lane * L::kXS + 4 * k) =
                make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
          __syncwarp();
          float acc[kCols];
#pragma unroll
          for (int e = 0; e < kCols; ++e) acc[e] = 0.0f;
#pragma unroll
          for (int r = 0; r < Cp; ++r) {
            const float* src = xp + (gw * Cp + r) * L::kXS + p * kCols;
            if constexpr (kCols % 4 == 0) {
#pragma unroll
              for (int e = 0; e < kCols; e += 4) {
                const float4 t = *reinterpret_cast<const float4*>(src + e);
                acc[e] += t.x;
                acc[e + 1] += t.y;
                acc[e + 2] += t.z;
                acc[e + 3] += t.w;
              }
            } else if constexpr (kCols == 2) {
              const float2 t = *reinterpret_cast<const float2*>(src);
              acc[0] += t.x;
              acc[1] += t.y;
            } else {
#pragma unroll
              for (int e = 0; e < kCols; ++e) acc[e] += src[e];
            }
          }
          if (g < G) {
            float* dst = mass + (bh * G + g) * nK;
#pragma unroll
            for (int e = 0; e < kCols; ++e) {
              const int b = col0 + 16 * ch + p * kCols + e;
              if (b < nK) dst[b] = acc[e];
            }
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (tid == 0 && *abort_flag) atomicCAS(status, 0, kStatusTimeout);
  if (warp == kMma) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

template <int D, int Cp>
int launch_mass(const ScoreLaunch& s, int nK, int BH, cudaStream_t stream) {
  using L = MassLayout<D>;
  CUtensorMap thi, tlo;
  if (!make_bf16_map(&thi, s.kbar_hi, BH, nK, D, 128) || !make_bf16_map(&tlo, s.kbar_lo, BH, nK, D, 128)) return -1;
  {
    const cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(mass_kernel<D, Cp>), static_cast<int>(L::kAlloc));
    if (e != cudaSuccess) return static_cast<int>(e);
  }
  constexpr int gpt = 128 / Cp;
  mass_kernel<D, Cp><<<dim3((s.G + gpt - 1) / gpt, BH), kMassThreads, L::kAlloc, stream>>>(
      thi, tlo, s.centroids, s.counts, s.N, s.Bk, nK, s.G, s.C, s.scale * 1.4426950408889634f, s.mass, s.status);
  return static_cast<int>(cudaGetLastError());
}

template <int D>
int launch_mass_any(const ScoreLaunch& s, int nK, int BH, cudaStream_t stream) {
  int Cp = 1;
  while (Cp < s.C) Cp <<= 1;
  switch (Cp) {
    case 1: return launch_mass<D, 1>(s, nK, BH, stream);
    case 2: return launch_mass<D, 2>(s, nK, BH, stream);
    case 4: return launch_mass<D, 4>(s, nK, BH, stream);
    case 8: return launch_mass<D, 8>(s, nK, BH, stream);
    default: return launch_mass<D, 16>(s, nK, BH, stream);
  }
}

static_assert(KtLayout<8>::kAllocFused <= 227 * 1024 && KtLayout<8>::kAlloc < KtLayout<8>::kAllocFused,
              "the fused k-means must fit the shared memory of one CTA");
static_assert(KtLayout<16>::kAlloc <= 227 * 1024 && KtLayout<16>::kAlloc < KtLayout<16>::kAllocFused,
              "C' = 16 runs without the key-mean warps");

// The tensor-core k-means over the groups of at most 128 rows (d = 128, C <= 16);
// with `fused` (C <= 8) the same launch also writes the key means (kbar hi / lo).
cudaError_t launch_kmeans_tc(const ScoreLaunch& s, int BH, int nK, bool fused, cudaStream_t stream) {
  CUtensorMap tq;
  if (!make_bf16_map(&tq, s.q, BH, s.N, 128, 128)) return cudaErrorInvalidValue;
  const long long items = static_cast<long long>(BH) * s.G;
  const int grid = static_cast<int>(items < s.num_sms ? items : s.num_sms);
  const uint16_t* kmat = static_cast<const uint16_t*>(s.k);
  if (s.C <= 8 && fused) {
    using L = KtLayout<8>;
    const cudaError_t e =
        ensure_smem_attr(reinterpret_cast<const void*>(kmeans_tc_kernel<8, true>), static_cast<int>(L::kAllocFused));
    if (e != cudaSuccess) return e;
    kmeans_tc_kernel<8, true><<<grid, kKtThreadsFused, L::kAllocFused, stream>>>(
        tq, BH, s.N, s.G, s.q_block, s.q_offsets, s.C, s.iters, s.centroids, s.counts, kWaitTimeoutNs, s.status,
        kmat, s.Bk, nK, s.kbar_hi, s.kbar_lo, s.kb_next);
  } else if (s.C <= 8) {
    using L = KtLayout<8>;
    const cudaError_t e =
        ensure_smem_attr(reinterpret_cast<const void*>(kmeans_tc_kernel<8, false>), static_cast<int>(L::kAlloc));
    if (e != cudaSuccess) return e;
    kmeans_tc_kernel<8, false><<<grid, kKtThreads, L::kAlloc, stream>>>(
        tq, BH, s.N, s.G, s.q_block, s.q_offsets, s.C, s.iters, s.centroids, s.counts, kWaitTimeoutNs, s.status,
        kmat, s.Bk, nK, s.kbar_hi, s.kbar_lo, s.kb_next);
  } else {
    using L = KtLayout<16>;
    const cudaError_t e =
        ensure_smem_attr(reinterpret_cast<const void*>(kmeans_tc_kernel<16, false>), static_cast<int>(L::kAlloc));
    if (e != cudaSuccess) return e;
    kmeans_tc_kernel<16, false><<<grid, kKtThreads, L::kAlloc, stream>>>(
        tq, BH, s.N, s.G, s.q_block, s.q_offsets, s.C, s.iters, s.centroids, s.counts, kWaitTimeoutNs, s.status,
        kmat, s.Bk, nK, s.kbar_hi, s.kbar_lo, s.kb_next);
  }
  return cudaGetLastError();
}

template <int D>
int launch_score_d(const ScoreLaunch& s, cudaStream_t stream) {
  const int BH = s.B * s.H;
  const int nK = (s.N + s.Bk - 1) / s.Bk;
  cudaError_t e = cudaSuccess;
  // the key means have their own launch unless the tensor-core k-means
  // (d = 128, C <= 8) computes them alongside, taking blocks from *kb_next;
  // key_means_rest_kernel then takes the blocks left (block indices are int:
  // layers of 2^30 key blocks and more keep the separate launch)
  const bool fused = D == 128 && s.C <= 8 && static_cast<int64_t>(BH) * nK < (int64_t{1} << 30);
  if (fused) {
    e = cudaMemsetAsync(s.kb_next, 0, sizeof(uint32_t), stream);
  } else {
    key_means_kernel<D><<<dim3((nK + 7) / 8, BH), kScoreThreads, 0, stream>>>(static_cast<const uint16_t*>(s.k),
                                                                              s.N, s.Bk, nK, s.kbar_hi, s.kbar_lo);
    e = cudaGetLastError();
  }
  if (e != cudaSuccess) return static_cast<int>(e);
  // groups of at most 128 rows (every group of the uniform layouts) take the
  // tensor-core k-means when d = 128 and C <= 16; the rest, the per-warp one
  int warp_min_rows = 0;
  if (D == 128 && s.C <= 16) {
    e = launch_kmeans_tc(s, BH, nK, fused, stream);
    if (e != cudaSuccess) return static_cast<int>(e);
    if (fused) {
      key_means_rest_kernel<D><<<s.num_sms * 8, kScoreThreads, 0, stream>>>(
          static_cast<const uint16_t*>(s.k), s.N, s.Bk, nK, BH * nK, s.kbar_hi, s.kbar_lo, s.kb_next);
      e = cudaGetLastError();
      if (e != cudaSuccess) return static_cast<int>(e);
    }
    warp_min_rows = 128;
    if (!s.q_offsets && s.q_block <= 128) return launch_mass_any<D>(s, nK, BH, stream);
  }
  using KL = KmLayout<D>;
  int km_blocks_per_sm[2] = {0, 0};
  e = ensure_smem_attr(reinterpret_cast<const void*>(kmeans_warp_kernel<D, 1>), static_cast<int>(KL::kAlloc));
  if (e == cudaSuccess)
    e = ensure_smem_attr(reinterpret_cast<const void*>(kmeans_warp_kernel<D, 2>), static_cast<int>(KL::kAlloc));
  if (e == cudaSuccess)
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&km_blocks_per_sm[0], kmeans_warp_kernel<D, 1>, kKmWarps * 32,
                                                      KL::kAlloc);
  if (e == cudaSuccess)
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&km_blocks_per_sm[1], kmeans_warp_kernel<D, 2>, kKmWarps * 32,
                                                      KL::kAlloc);
  if (e != cudaSuccess) return static_cast<int>(e);
  if (km_blocks_per_sm[0] < 1 || km_blocks_per_sm[1] < 1) return static_cast<int>(cudaErrorInvalidConfiguration);
  {
    // a persistent grid: every warp walks groups with a stride of the grid's warps
    const long long items = static_cast<long long>(BH) * s.G;
    const int per_sm = s.C <= 8 ? km_blocks_per_sm[0] : km_blocks_per_sm[1];
    const long long want = (items + kKmWarps - 1) / kKmWarps;
    const int grid = static_cast<int>(want < static_cast<long long>(s.num_sms) * per_sm
                                          ? want
                                          : static_cast<long long>(s.num_sms) * per_sm);
    if (s.C <= 8)
      kmeans_warp_kernel<D, 1><<<grid, kKmWarps * 32, KL::kAlloc, stream>>>(
          static_cast<const uint16_t*>(s.q), BH, s.N, s.G, s.q_block, s.q_offsets, s.C, s.iters, s.centroids,
          s.counts, warp_min_rows, s.status);
    else
      kmeans_warp_kernel<D, 2><<<grid, kKmWarps * 32, KL::kAlloc, stream>>>(
          static_cast<const uint16_t*>(s.q), BH, s.N, s.G, s.q_block, s.q_offsets, s.C, s.iters, s.centroids,
          s.counts, warp_min_rows, s.status);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return static_cast<int>(e);
  return launch_mass_any<D>(s, nK, BH, stream);
}

}  // namespace

size_t score_workspace_bytes(int B, int H, int N, int D, int G, int Bk, int C) {
  const size_t BH = static_cast<size_t>(B) * H;
  const size_t nK = (static_cast<size_t>(N) + Bk - 1) / Bk;
  auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  return up(BH * nK * D * 4) + up(BH * G * C * D * 4) + up(BH * G * C * 4) + up(sizeof(uint32_t));
}

int launch_score(const ScoreLaunch& s, cudaStream_t stream) {
  if (s.D == 128) return launch_score_d<128>(s, stream);
  if (s.D == 64) return launch_score_d<64>(s, stream);
  return -1;
}

}  // namespace isa_impl
