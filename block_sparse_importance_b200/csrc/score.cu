// IBCS block scorer.
//
// "AB-Attention: Accurate Block Attention for Accelerating Video Diffusion
// Transformers", Intra-Block Clustering Selector: similar queries are
// grouped only within each query block, each group gets a representative and
// a weight equal to its size, and the representatives score small key blocks
// without reordering tokens.  Key blocks are summarised by their means.
//
// Three kernels:
//   key_means_kernel  kbar_b = mean of the valid rows of key block b (fp32);
//   kmeans_kernel     per (batch*head, group): Lloyd's k-means, centroids
//                     initialised at rows floor(c n / C), `iters` rounds of
//                     nearest-centroid assignment (squared distance, ties to
//                     the lower c) and mean update; rows stream through
//                     shared memory 128 at a time;
//   mass_kernel       per (batch*head, 128 / C' groups): logits
//                     l = scale mu_c . kbar_b + ln L_b, a first pass for the
//                     per-centroid softmax max and sum over all key blocks, a
//                     second pass for mass_b = sum_c n_c exp(l - max_c) / sum_c.

#include <cuda_bf16.h>

#include <cstdint>

#include "isa_internal.h"

namespace isa_impl {
namespace {

constexpr int kScoreThreads = 256;
constexpr int kChunkRows = 128;
constexpr int kMassRows = 128;    // centroid rows per mass CTA
constexpr int kMassBlocks = 64;   // key blocks per smem chunk

__device__ __forceinline__ float bf16_to_f(uint16_t h) { return __uint_as_float(static_cast<uint32_t>(h) << 16); }

// ------------------------------------------------------------ key means
template <int D>
__global__ void __launch_bounds__(kScoreThreads) key_means_kernel(const uint16_t* __restrict__ k, int N, int Bk,
                                                                  int nK, float* __restrict__ kbar) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.x * (kScoreThreads / 32) + warp;
  const int64_t bh = blockIdx.y;
  if (b >= nK) return;
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
  float* o = kbar + (bh * nK + b) * D + lane * PER;
#pragma unroll
  for (int i = 0; i < PER; ++i) o[i] = acc[i] * inv;
}

// ---------------------------------------------------------------- k-means
template <int D>
__global__ void __launch_bounds__(kScoreThreads) kmeans_kernel(const uint16_t* __restrict__ q, int N, int G,
                                                               int q_block, const int32_t* __restrict__ off, int C,
                                                               int iters, float* __restrict__ centroids,
                                                               int32_t* __restrict__ counts, int* status) {
  extern __shared__ __align__(16) uint8_t sm[];
  uint16_t* rows = reinterpret_cast<uint16_t*>(sm);                       // [128][D]
  float* mu = reinterpret_cast<float*>(sm + kChunkRows * D * 2);           // [C][D]
  float* sums = mu + C * D;                                                // [C][D]
  int* cnt = reinterpret_cast<int*>(sums + C * D);                        // [C]
  int* assign = cnt + 16;                                                  // [128]
  const int g = blockIdx.x;
  const int64_t bh = blockIdx.y;
  const int tid = threadIdx.x;
  int r0, r1;
  if (off) {
    r0 = off[g];
    r1 = off[g + 1];
    if (r0 < 0 || r1 > N || r1 <= r0) {  // malformed offsets: leave an empty group
      if (tid == 0) atomicCAS(status, 0, kStatusDeviceCheck);
      r1 = r0 = 0;
    }
  } else {
    r0 = g * q_block;
    r1 = min(N, r0 + q_block);
  }
  const int n = r1 - r0;
  const uint16_t* qg = q + (bh * N + r0) * D;
  for (int i = tid; i < C * D; i += kScoreThreads) {
    const int c = i / D, j = i - c * D;
    const int r = static_cast<int>((static_cast<int64_t>(c) * n) / C);
    mu[i] = n > 0 ? bf16_to_f(qg[static_cast<int64_t>(r) * D + j]) : 0.0f;
  }
  const bool one_chunk = n <= kChunkRows;
  for (int it = 0; it < iters; ++it) {
    for (int i = tid; i < C * D; i += kScoreThreads) sums[i] = 0.0f;
    if (tid < 16) cnt[tid] = 0;
    __syncthreads();
    for (int cs = 0; cs < n; cs += kChunkRows) {
      const int rc = min(kChunkRows, n - cs);
      if (!(one_chunk && it > 0)) {
        const uint4* src = reinterpret_cast<const uint4*>(qg + static_cast<int64_t>(cs) * D);
        uint4* dst = reinterpret_cast<uint4*>(rows);
        for (int i = tid; i < rc * D / 8; i += kScoreThreads) dst[i] = src[i];
      }
      __syncthreads();
      // assignment: two threads per row, each summing half of the columns
      {
        const int r = tid >> 1, half = tid & 1;
        int best_c = 0;
        float best = INFINITY;
        for (int c = 0; c < C; ++c) {
          float part = 0.0f;
          if (r < rc) {
            const uint16_t* x = rows + r * D + half * (D / 2);
            const float* m = mu + c * D + half * (D / 2);
#pragma unroll 16
            for (int j = 0; j < D / 2; ++j) {
              const float t = bf16_to_f(x[j]) - m[j];
              part = fmaf(t, t, part);
            }
          }
          const float dist = part + __shfl_xor_sync(0xffffffffu, part, 1);
          if (dist < best) {
            best = dist;
            best_c = c;
          }
        }
        if (r < rc && half == 0) assign[r] = best_c;
      }
      __syncthreads();
      // accumulate rows into their cluster sums: thread = (column, half of rows)
      {
        constexpr int kColThreads = D;
        const int j = tid % kColThreads, part = tid / kColThreads, nparts = kScoreThreads / kColThreads;
        float acc[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) acc[c] = 0.0f;
        for (int r = part; r < rc; r += nparts) {
          const float v = bf16_to_f(rows[r * D + j]);
          const int a = assign[r];
#pragma unroll
          for (int c = 0; c < 16; ++c) acc[c] += (a == c) ? v : 0.0f;
        }
#pragma unroll
        for (int c = 0; c < 16; ++c)
          if (c < C) atomicAdd(&sums[c * D + j], acc[c]);
        for (int r = tid; r < rc; r += kScoreThreads) atomicAdd(&cnt[assign[r]], 1);
      }
      __syncthreads();
    }
    for (int i = tid; i < C * D; i += kScoreThreads) {
      const int c = i / D;
      if (cnt[c] > 0) mu[i] = sums[i] / static_cast<float>(cnt[c]);
    }
    __syncthreads();
  }
  const int64_t t = bh * G + g;
  for (int i = tid; i < C * D; i += kScoreThreads) centroids[t * C * D + i] = mu[i];
  if (tid < C) counts[t * C + tid] = cnt[tid];
}

// ------------------------------------------------------------------ mass
// Rows of the CTA: group gl (0 .. 128/Cp - 1) owns rows [gl*Cp, gl*Cp + C)
// with Cp = C rounded up to a power of two; padding rows carry count 0.
// Thread t: row slab rs = t / 16 (8 rows), block lane bl = t % 16 (4 blocks
// of each 64-block chunk).
template <int D, int Cp>
__global__ void __launch_bounds__(kScoreThreads) mass_kernel(const float* __restrict__ centroids,
                                                             const int32_t* __restrict__ counts,
                                                             const float* __restrict__ kbar, int N, int Bk,
                                                             int nK, int G, int C, float scale,
                                                             float* __restrict__ mass) {
  extern __shared__ __align__(16) uint8_t sm[];
  constexpr int KP = D + 4;  // padded row stride of the key chunk (floats)
  float* cen = reinterpret_cast<float*>(sm);               // [128][D]
  float* kb = cen + kMassRows * D;                          // [64][KP]
  float* stat_m = kb + kMassBlocks * KP;                    // [128]
  float* stat_z = stat_m + kMassRows;                       // [128]
  float* wgt = stat_z + kMassRows;                          // [128] n_c (0 for padding)
  const int tid = threadIdx.x;
  const int64_t bh = blockIdx.y;
  const int gpc = kMassRows / Cp;
  const int g0 = blockIdx.x * gpc;
  for (int i = tid; i < kMassRows; i += kScoreThreads) {
    const int gl = i / Cp, c = i - gl * Cp, g = g0 + gl;
    wgt[i] = (c < C && g < G) ? static_cast<float>(counts[(bh * G + g) * C + c]) : 0.0f;
  }
  for (int i = tid; i < kMassRows * D; i += kScoreThreads) {
    const int rr = i / D, j = i - rr * D;
    const int gl = rr / Cp, c = rr - gl * Cp, g = g0 + gl;
    cen[i] = (c < C && g < G) ? centroids[((bh * G + g) * C + c) * D + j] : 0.0f;
  }
  const int rs = tid >> 4, bl = tid & 15;
  float run_m[8], run_z[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    run_m[i] = -INFINITY;
    run_z[i] = 0.0f;
  }
  const float* kbh = kbar + bh * nK * D;
  for (int pass = 0; pass < 2; ++pass) {
    if (pass == 1) {
      // combine the 16 partial (max, sum) of each row and publish them
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float m = run_m[i], z = run_z[i];
#pragma unroll
        for (int o = 1; o < 16; o <<= 1) {
          const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
          const float z2 = __shfl_xor_sync(0xffffffffu, z, o);
          const float mm = fmaxf(m, m2);
          z = (mm == -INFINITY) ? 0.0f : z * __expf(m - mm) + z2 * __expf(m2 - mm);
          m = mm;
        }
        if (bl == 0) {
          stat_m[rs * 8 + i] = m;
          stat_z[rs * 8 + i] = z;
        }
      }
    }
    for (int cb = 0; cb < nK; cb += kMassBlocks) {
      __syncthreads();
      for (int i = tid; i < kMassBlocks * D / 4; i += kScoreThreads) {
        const int b = i / (D / 4), j4 = i - b * (D / 4);
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (cb + b < nK) v = reinterpret_cast<const float4*>(kbh + static_cast<int64_t>(cb + b) * D)[j4];
        float* dst = kb + b * KP + 4 * j4;
        dst[0] = v.x;
        dst[1] = v.y;
        dst[2] = v.z;
        dst[3] = v.w;
      }
      __syncthreads();
      float acc[8][4];
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int u = 0; u < 4; ++u) acc[i][u] = 0.0f;
      for (int j = 0; j < D; j += 4) {
        float4 kv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) kv[u] = *reinterpret_cast<const float4*>(kb + (bl * 4 + u) * KP + j);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float4 cv = *reinterpret_cast<const float4*>(cen + (rs * 8 + i) * D + j);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            acc[i][u] = fmaf(cv.x, kv[u].x, acc[i][u]);
            acc[i][u] = fmaf(cv.y, kv[u].y, acc[i][u]);
            acc[i][u] = fmaf(cv.z, kv[u].z, acc[i][u]);
            acc[i][u] = fmaf(cv.w, kv[u].w, acc[i][u]);
          }
        }
      }
      float lnL[4];
      bool ok[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int b = cb + bl * 4 + u;
        ok[u] = b < nK;
        lnL[u] = ok[u] ? logf(static_cast<float>(min(Bk, N - b * Bk))) : 0.0f;
      }
      if (pass == 0) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            if (!ok[u]) continue;
            const float l = fmaf(scale, acc[i][u], lnL[u]);
            if (l > run_m[i]) {
              run_z[i] = run_z[i] * __expf(run_m[i] - l) + 1.0f;
              run_m[i] = l;
            } else {
              run_z[i] += __expf(l - run_m[i]);
            }
          }
        }
      } else {
        // rows of this thread: 8 consecutive rows = 8/Cp whole groups (Cp <= 8)
        // or half of a 16-row group (Cp == 16, combined with the partner slab)
        float part[4][8];
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int i = 0; i < 8; ++i) part[u][i] = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int rr = rs * 8 + i;
          const float w = wgt[rr];
          const float m = stat_m[rr], z = stat_z[rr];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float l = fmaf(scale, acc[i][u], lnL[u]);
            part[u][i] = (w > 0.0f && ok[u]) ? w * (__expf(l - m) / z) : 0.0f;
          }
        }
        if constexpr (Cp <= 8) {
#pragma unroll
          for (int s0 = 0; s0 < 8; s0 += Cp) {
            const int gl = (rs * 8 + s0) / Cp, g = g0 + gl;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              float sum = 0.0f;
#pragma unroll
              for (int i = s0; i < s0 + Cp; ++i) sum += part[u][i];
              const int b = cb + bl * 4 + u;
              if (g < G && ok[u]) mass[(bh * G + g) * nK + b] = sum;
            }
          }
        } else {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            float sum = 0.0f;
#pragma unroll
            for (int i = 0; i < 8; ++i) sum += part[u][i];
            sum += __shfl_xor_sync(0xffffffffu, sum, 16);
            const int gl = (rs * 8) / 16, g = g0 + gl, b = cb + bl * 4 + u;
            if ((rs & 1) == 0 && g < G && ok[u]) mass[(bh * G + g) * nK + b] = sum;
          }
        }
      }
    }
    __syncthreads();
  }
}

template <int D, int Cp>
int launch_mass(const ScoreLaunch& s, int nK, int BH, cudaStream_t stream) {
  constexpr int gpc = kMassRows / Cp;
  const size_t ms_smem = (kMassRows * D + kMassBlocks * (D + 4) + 3 * kMassRows) * 4;
  static bool ms_attr = false;
  if (!ms_attr) {
    cudaError_t e = cudaFuncSetAttribute(mass_kernel<D, Cp>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(ms_smem));
    if (e != cudaSuccess) return static_cast<int>(e);
    ms_attr = true;
  }
  mass_kernel<D, Cp><<<dim3((s.G + gpc - 1) / gpc, BH), kScoreThreads, ms_smem, stream>>>(
      s.centroids, s.counts, s.kbar, s.N, s.Bk, nK, s.G, s.C, s.scale, s.mass);
  return static_cast<int>(cudaGetLastError());
}

template <int D>
int launch_score_d(const ScoreLaunch& s, cudaStream_t stream) {
  const int BH = s.B * s.H;
  const int nK = (s.N + s.Bk - 1) / s.Bk;
  key_means_kernel<D><<<dim3((nK + 7) / 8, BH), kScoreThreads, 0, stream>>>(static_cast<const uint16_t*>(s.k), s.N,
                                                                            s.Bk, nK, s.kbar);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return static_cast<int>(e);
  const size_t km_smem = kChunkRows * D * 2 + 2 * s.C * D * 4 + (16 + kChunkRows) * 4;
  static bool km_attr = false;
  if (!km_attr) {
    e = cudaFuncSetAttribute(kmeans_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, 64 * 1024 + 16 * 1024);
    if (e != cudaSuccess) return static_cast<int>(e);
    km_attr = true;
  }
  kmeans_kernel<D><<<dim3(s.G, BH), kScoreThreads, km_smem, stream>>>(static_cast<const uint16_t*>(s.q), s.N, s.G,
                                                                      s.q_block, s.q_offsets, s.C, s.iters,
                                                                      s.centroids, s.counts, s.status);
  e = cudaGetLastError();
  if (e != cudaSuccess) return static_cast<int>(e);
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

}  // namespace

size_t score_workspace_bytes(int B, int H, int N, int D, int G, int Bk, int C) {
  const size_t BH = static_cast<size_t>(B) * H;
  const size_t nK = (static_cast<size_t>(N) + Bk - 1) / Bk;
  auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  return up(BH * nK * D * 4) + up(BH * G * C * D * 4) + up(BH * G * C * 4);
}

int launch_score(const ScoreLaunch& s, cudaStream_t stream) {
  if (s.D == 128) return launch_score_d<128>(s, stream);
  if (s.D == 64) return launch_score_d<64>(s, stream);
  return -1;
}

}  // namespace isa_impl
