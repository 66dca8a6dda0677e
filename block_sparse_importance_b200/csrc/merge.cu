// Tail merging of the permuted layout's last query tiles.
//
// "iCATS: Fast Video Generation via Interaction-Aware Sparse Attention and
// Timestep-Adaptive Sparsity", AI summary, "Approach": the tail blocks of query
// clusters are merged with Hamming-nearest compatible clusters, to cut the
// padding of their last tiles.  The schedule, per (batch, head):
//   * the tail of cluster g is its last t_g = n_g mod 128 rows (all of it when
//     n_g < 128); in a merged tile it takes a slot of ceil(t_g / 32) * 32 rows
//     (whole quarters: the 32 rows one softmax warp handles share one plan),
//     members packed from row 0 in the order they joined;
//   * tails are taken by decreasing t_g, ties to the lower g;
//   * a tail may join an open tile when its slot fits, the tile has fewer
//     than 4 members, and the union U of the members' plan blocks with the
//     tail's plan P added needs fewer KV tiles of 128 / Bk blocks than U and P
//     apart; it joins the one whose U is nearest to P in Hamming distance
//     (ties to the tile opened first), else it opens a tile;
//   * every row keeps its own cluster's plan and log-weights: a merged tile
//     runs the blocks of U ascending, and a block outside a row's plan carries
//     log-weight -inf for that row (the table built here).
// Plan rows are taken to hold distinct blocks, as the selector writes them.
//
// Kernels:
//   tail_merge_kernel   one CTA per (b, h): the greedy schedule (plan masks of
//                       nK bits, union masks in shared memory when they fit,
//                       else in the workspace), then each merged tile's union
//                       list and log-weight table;
//   merge_items_kernel  one CTA per (b, h): the attention's work items: the
//                       full tiles of every cluster, then the head's tiles of
//                       tails (a single tail runs on its own plan row).

#include <cstdint>

#include "isa_internal.h"

namespace isa_impl {
namespace {

constexpr int kMergeThreads = 256;
constexpr int kMergeWarps = kMergeThreads / 32;
constexpr int kTileRowsM = 128;

__device__ __forceinline__ int kv_tiles(int n, int b) { return (n + b - 1) / b; }

__device__ __forceinline__ uint64_t block_min_u64(uint64_t v, uint64_t* red) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const uint64_t x = __shfl_xor_sync(0xffffffffu, v, o);
    v = x < v ? x : v;
  }
  __syncthreads();
  if (lane == 0) red[w] = v;
  __syncthreads();
  uint64_t r = red[0];
#pragma unroll
  for (int i = 1; i < kMergeWarps; ++i) r = red[i] < r ? red[i] : r;
  return r;
}

__global__ void __launch_bounds__(kMergeThreads) tail_merge_kernel(MergeLaunch m) {
  // the greedy's state: per tile rows, members and union size, the union
  // masks and the two plan masks (the tail's, and the next tail's being
  // built), in shared memory when they fit, else in the workspace
  extern __shared__ __align__(16) uint32_t dyn[];
  __shared__ uint64_t red[kMergeWarps];
  __shared__ int s_n_tails, s_n_bins;
  __shared__ int cnt[kTileRowsM];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t bh = blockIdx.x;
  const int G = m.G, S = m.S, W = m.W, b = kTileRowsM / m.Bk;
  const int32_t* off = m.q_offsets;
  const int32_t* idx = m.idx + bh * G * S;
  const float* lw = m.log_w + bh * G * S;
  MergeBin* bins = m.bins + bh * G;
  int32_t* order = m.order + bh * G;
  uint32_t* st = m.state_in_smem ? dyn : m.state + bh * merge_state_words(G, W);
  int32_t* b_rows = reinterpret_cast<int32_t*>(st);
  int32_t* b_n = b_rows + G;
  int32_t* b_ulen = b_n + G;
  uint32_t* Pbuf = st + 3 * G;  // two plan masks of W words
  uint32_t* U = Pbuf + 2 * W;   // [G][W]
  int32_t* units = m.unions + bh * static_cast<int64_t>(G) * S;
  float* table = m.tables + bh * static_cast<int64_t>(4) * G * S;

  // ---- the tails, by decreasing rows, ties to the lower cluster
  for (int i = tid; i < kTileRowsM; i += kMergeThreads) cnt[i] = 0;
  for (int w = tid; w < 2 * W; w += kMergeThreads) Pbuf[w] = 0u;
  __syncthreads();
  for (int g = tid; g < G; g += kMergeThreads) {
    const int t = (off[g + 1] - off[g]) % kTileRowsM;
    if (t > 0) atomicAdd(&cnt[t], 1);
  }
  __syncthreads();
  if (tid == 0) {
    int pos = 0;
    for (int t = kTileRowsM - 1; t >= 1; --t) {  // start of each row count's run
      const int c = cnt[t];
      cnt[t] = pos;
      pos += c;
    }
    s_n_tails = pos;
    for (int g = 0; g < G; ++g) {
      const int t = (off[g + 1] - off[g]) % kTileRowsM;
      if (t > 0) order[cnt[t]++] = g;
    }
    s_n_bins = 0;
  }
  __syncthreads();
  const int n_tails = s_n_tails;

  // this thread's entries of a tail's plan, loaded a step ahead of their use
  constexpr int kPre = 4;
  int pv[kPre];
  auto load_plan = [&](int i) {
    const int g = order[i];
#pragma unroll
    for (int q = 0; q < kPre; ++q) {
      const int s = tid + q * kMergeThreads;
      pv[q] = s < S ? idx[static_cast<int64_t>(g) * S + s] : -1;
    }
  };
  auto set_plan = [&](int i, uint32_t* P) {
    const int g = order[i];
    int q = 0;
    for (int s = tid; s < S; s += kMergeThreads, ++q) {
      const int blk = q < kPre ? pv[q] : idx[static_cast<int64_t>(g) * S + s];
      if (blk >= 0 && blk < m.nK) {
        atomicOr(&P[blk >> 5], 1u << (blk & 31));
      } else {
        atomicCAS(m.status, 0, kStatusDeviceCheck);
      }
    }
  };
  if (n_tails > 0) {
    load_plan(0);
    set_plan(0, Pbuf);
  }
  __syncthreads();

  // ---- the greedy schedule
  for (int i = 0; i < n_tails; ++i) {
    uint32_t* P = Pbuf + (i & 1) * W;
    uint32_t* Pn = Pbuf + ((i + 1) & 1) * W;
    const int g = order[i];
    const int t = (off[g + 1] - off[g]) % kTileRowsM;
    const int slot = (t + 31) / 32 * 32;
    if (i + 1 < n_tails) load_plan(i + 1);
    const int n_bins = s_n_bins;
    uint64_t key = ~0ull;  // (Hamming distance, tile): the smallest wins
    for (int k = tid; k < n_bins; k += kMergeThreads) {
      if (b_rows[k] + slot > kTileRowsM || b_n[k] >= 4) continue;
      const uint32_t* Uk = U + static_cast<int64_t>(k) * W;
      int inter = 0;
      for (int w = 0; w < W; ++w) inter += __popc(Uk[w] & P[w]);
      const int ul = b_ulen[k], un = ul + S - inter;
      if (kv_tiles(un, b) >= kv_tiles(ul, b) + kv_tiles(S, b)) continue;
      const uint64_t ham = static_cast<uint64_t>(ul + S - 2 * inter);
      const uint64_t kk = (ham << 32) | static_cast<uint32_t>(k);
      key = kk < key ? kk : key;
    }
    for (int w = tid; w < W; w += kMergeThreads) Pn[w] = 0u;  // read last in step i - 1
    key = block_min_u64(key, red);  // (its barriers also order the clearing before the next plan's bits)
    int k;
    if (key != ~0ull) {
      k = static_cast<int>(key & 0xFFFFFFFFu);
      if (tid == 0) {
        const int ham = static_cast<int>(key >> 32);
        const int inter = (b_ulen[k] + S - ham) / 2;
        const int n = b_n[k];
        bins[k].g[n] = g;
        bins[k].slot[n] = b_rows[k];
        b_n[k] = n + 1;
        b_rows[k] += slot;
        b_ulen[k] += S - inter;
      }
      uint32_t* Uk = U + static_cast<int64_t>(k) * W;
      for (int w = tid; w < W; w += kMergeThreads) Uk[w] |= P[w];
    } else {
      k = n_bins;
      if (tid == 0) {
        b_n[k] = 1;
        b_rows[k] = slot;
        b_ulen[k] = S;
        for (int j = 0; j < 4; ++j) {
          bins[k].g[j] = j == 0 ? g : -1;
          bins[k].slot[j] = j == 0 ? 0 : -1;
        }
        s_n_bins = n_bins + 1;
      }
      uint32_t* Uk = U + static_cast<int64_t>(k) * W;
      for (int w = tid; w < W; w += kMergeThreads) Uk[w] = P[w];
    }
    if (i + 1 < n_tails) set_plan(i + 1, Pn);
    __syncthreads();
  }
  const int n_bins = s_n_bins;
  for (int k = tid; k < n_bins; k += kMergeThreads) {
    bins[k].n = b_n[k];
    bins[k].rows = b_rows[k];
    bins[k].ulen = b_ulen[k];
    bins[k].uoff = -1;
    bins[k].toff = -1;
  }
  __syncthreads();

  // ---- union lists and log-weight tables of the merged tiles (2+ members)
  if (tid == 0) {
    int uo = 0, to = 0, multi = 0;
    for (int k = 0; k < n_bins; ++k) {
      MergeBin& bn = bins[k];
      if (bn.n > 1) {
        bn.uoff = uo;
        bn.toff = to;
        uo += bn.ulen;
        to += bn.n * bn.ulen;
        ++multi;
      }
    }
    m.counts[2 * bh] = n_bins;
    m.counts[2 * bh + 1] = multi;
  }
  __syncthreads();
  int32_t* pre = m.prefix + (bh * kMergeWarps + warp) * static_cast<int64_t>(W);  // this warp's scratch
  for (int k = warp; k < n_bins; k += kMergeWarps) {
    const MergeBin bn = bins[k];
    if (bn.n < 2) continue;
    const uint32_t* Uk = U + static_cast<int64_t>(k) * W;
    // exclusive prefix of the union's set bits over the mask words
    int carry = 0;
    for (int c0 = 0; c0 < W; c0 += 32) {
      const int w = c0 + lane;
      const int cw = w < W ? __popc(Uk[w]) : 0;
      int inc = cw;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int x = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += x;
      }
      if (w < W) pre[w] = carry + inc - cw;
      carry += __shfl_sync(0xffffffffu, inc, 31);
    }
    __syncwarp();
    // the union, ascending
    for (int w = lane; w < W; w += 32) {
      uint32_t bits = Uk[w];
      int p = pre[w];
      while (bits) {
        units[bn.uoff + p++] = w * 32 + __ffs(static_cast<int>(bits)) - 1;
        bits &= bits - 1;
      }
    }
    // per member: its log-weight at each union position, -inf off its plan
    for (int e = lane; e < bn.n * bn.ulen; e += 32) table[bn.toff + e] = -INFINITY;
    __syncwarp();
    for (int j = 0; j < bn.n; ++j) {
      const int g = bn.g[j];
      for (int s = lane; s < S; s += 32) {
        const int blk = idx[static_cast<int64_t>(g) * S + s];
        if (blk < 0 || blk >= m.nK) continue;  // flagged above
        const int w = blk >> 5;
        const int pos = pre[w] + __popc(Uk[w] & ((1u << (blk & 31)) - 1u));
        table[bn.toff + j * bn.ulen + pos] = lw[static_cast<int64_t>(g) * S + s];
      }
    }
    __syncwarp();
  }
}

// The attention's work items.  All heads' merged tiles come first, each
// head's by decreasing union length (so that the two tiles a CTA runs side by
// side have about as many KV tiles); then every head's clusters in order, each
// with its full 128-row tiles and, when its tail was not merged, the tail
// (neighbouring tiles of one cluster share their K/V stream when a CTA runs
// them as a pair).  One CTA per (b, h); CTA 0 writes the total.
__global__ void __launch_bounds__(kMergeThreads) merge_items_kernel(MergeLaunch m) {
  __shared__ int s_red[kMergeThreads];
  const int tid = threadIdx.x;
  const int bh = blockIdx.x;
  const int G = m.G;
  const int32_t* off = m.q_offsets;
  auto block_sum = [&](int v) -> int {
    s_red[tid] = v;
    __syncthreads();
    for (int d = kMergeThreads / 2; d > 0; d >>= 1) {
      if (tid < d) s_red[tid] += s_red[tid + d];
      __syncthreads();
    }
    const int r = s_red[0];
    __syncthreads();
    return r;
  };
  // full tiles per head (the same for every head), merged tiles of all heads
  // and of the heads before this one, single tails before this head's
  int full = 0;
  for (int g = tid; g < G; g += kMergeThreads) full += (off[g + 1] - off[g]) / kTileRowsM;
  int multi_all = 0, multi_before = 0, single_before = 0, single_all = 0;
  for (int h = tid; h < m.BH; h += kMergeThreads) {
    const int nb = m.counts[2 * h], nm = m.counts[2 * h + 1];
    multi_all += nm;
    single_all += nb - nm;
    if (h < bh) {
      multi_before += nm;
      single_before += nb - nm;
    }
  }
  const int F = block_sum(full);
  multi_all = block_sum(multi_all);
  single_all = block_sum(single_all);
  multi_before = block_sum(multi_before);
  single_before = block_sum(single_before);
  const MergeBin* bins = m.bins + static_cast<int64_t>(bh) * G;
  const int nb = m.counts[2 * bh];
  // merged tiles, ranked by union length (longer first, ties by opening order)
  for (int k = tid; k < nb; k += kMergeThreads) {
    const MergeBin bn = bins[k];
    if (bn.n < 2) continue;
    int rank = 0;
    for (int k2 = 0; k2 < nb; ++k2) {
      const int n2 = bins[k2].n, u2 = bins[k2].ulen;
      if (n2 > 1 && (u2 > bn.ulen || (u2 == bn.ulen && k2 < k))) ++rank;
    }
    m.items[multi_before + rank] = WorkItem{bh, -1 - k, 0, bn.rows};
  }
  // the clusters whose tail runs alone (the tails' order array is free now)
  int32_t* alone = m.order + static_cast<int64_t>(bh) * G;
  for (int g = tid; g < G; g += kMergeThreads) alone[g] = 0;
  __syncthreads();
  for (int k = tid; k < nb; k += kMergeThreads)
    if (bins[k].n == 1) alone[bins[k].g[0]] = 1;
  __syncthreads();
  // this head's clusters: per-thread runs, placed by a block-wide scan
  WorkItem* it = m.items + multi_all + static_cast<int64_t>(bh) * F + single_before;
  const int per = (G + kMergeThreads - 1) / kMergeThreads;
  const int g0 = min(G, tid * per), g1 = min(G, g0 + per);
  int mine = 0;
  for (int g = g0; g < g1; ++g) mine += (off[g + 1] - off[g]) / kTileRowsM + alone[g];
  s_red[tid] = mine;
  __syncthreads();
  for (int d = 1; d < kMergeThreads; d <<= 1) {  // inclusive scan
    const int v = tid >= d ? s_red[tid - d] : 0;
    __syncthreads();
    s_red[tid] += v;
    __syncthreads();
  }
  int o = s_red[tid] - mine;
  for (int g = g0; g < g1; ++g) {
    const int nf = (off[g + 1] - off[g]) / kTileRowsM;
    for (int f = 0; f < nf; ++f) it[o++] = WorkItem{bh, g, off[g] + f * kTileRowsM, kTileRowsM};
    if (alone[g]) {
      const int t = (off[g + 1] - off[g]) % kTileRowsM;
      it[o++] = WorkItem{bh, g, off[g + 1] - t, t};
    }
  }
  if (bh == 0 && tid == 0) *m.item_count = multi_all + m.BH * F + single_all;
}

// The merged tiles of all heads, spread over the attention's persistent
// CTAs.  The grid takes the item pairs round-robin (pair p runs on CTA
// p mod grid), and merged tiles differ in length, so the pairs are ordered by
// length, longest first, and dealt to the CTAs in alternating direction, one
// round of `grid` pairs after another (the last, partial round in plain
// order); each pair holds two tiles of about the same length.  One CTA sorts
// (length, position) keys in shared memory (bitonic); more merged tiles than
// it holds keep the per-head order.
constexpr int kBalanceThreads = 1024;
constexpr int kBalanceMax = 8192;
constexpr size_t kBalanceSmem = static_cast<size_t>(kBalanceMax) * (8 + sizeof(WorkItem));
__global__ void __launch_bounds__(kBalanceThreads) merge_balance_kernel(MergeLaunch m) {
  extern __shared__ __align__(16) unsigned long long key[];  // [kBalanceMax], then the items
  WorkItem* stash = reinterpret_cast<WorkItem*>(key + kBalanceMax);
  __shared__ int s_n;
  const int tid = threadIdx.x;
  if (tid == 0) {
    int n = 0;
    for (int h = 0; h < m.BH; ++h) n += m.counts[2 * h + 1];
    s_n = n;
  }
  __syncthreads();
  const int n = s_n;
  if (n < 3 || n > kBalanceMax || m.grid < 2) return;
  const int b = kTileRowsM / m.Bk;
  int pow2 = 1;
  while (pow2 < n) pow2 <<= 1;
  for (int i = tid; i < pow2; i += kBalanceThreads) {
    if (i < n) {
      const WorkItem it = m.items[i];
      stash[i] = it;
      const int ulen = m.bins[static_cast<int64_t>(it.bh) * m.G + (-1 - it.g)].ulen;
      const unsigned T = static_cast<unsigned>((ulen + b - 1) / b);
      key[i] = (static_cast<unsigned long long>(0xFFFFFFFFu - T) << 32) | static_cast<unsigned>(i);
    } else {
      key[i] = ~0ull;  // sorts last
    }
  }
  __syncthreads();
  for (int size = 2; size <= pow2; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = tid; i < pow2; i += kBalanceThreads) {
        const int j = i ^ stride;
        if (j > i) {
          const bool up = (i & size) == 0;
          const unsigned long long a = key[i], c = key[j];
          if ((a > c) == up) {
            key[i] = c;
            key[j] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  // an odd last (shortest) tile stays last, paired with the first item after
  // the merged ones
  const int grid = m.grid;
  const int n2 = n & ~1, pairs = n2 / 2;
  const int full_rounds = pairs / grid;
  for (int i = tid; i < n; i += kBalanceThreads) {
    int pos = i;
    if (i < n2) {
      const int pr = i >> 1, r = pr / grid;
      int c = pr - r * grid;
      if ((r & 1) && r < full_rounds) c = grid - 1 - c;
      pos = 2 * (r * grid + c) + (i & 1);
    }
    m.items[pos] = stash[static_cast<int>(key[i] & 0xFFFFFFFFu)];
  }
}

}  // namespace

MergeCarve merge_carve(int BH, int N, int G, int S, int nK) {
  auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  const size_t bh = static_cast<size_t>(BH), g = static_cast<size_t>(G), s = static_cast<size_t>(S);
  const size_t w = (static_cast<size_t>(nK) + 31) / 32;
  MergeCarve c{};
  size_t o = 0;
  c.bins = o;
  o += up(bh * g * sizeof(MergeBin));
  c.counts = o;
  o += up(bh * 8);
  c.order = o;
  o += up(bh * g * 4);
  c.state = o;
  o += up(bh * merge_state_words(G, static_cast<int>(w)) * 4);
  c.prefix = o;
  o += up(bh * kMergeWarps * w * 4);
  c.unions = o;
  o += up(bh * g * s * 4);
  c.tables = o;
  o += up(bh * 4 * g * s * 4);
  c.items = o;
  o += up(bh * (static_cast<size_t>(N) / kTileRowsM + g) * sizeof(WorkItem));
  c.item_count = o;
  o += 256;
  c.total = o;
  return c;
}

int launch_tail_merge(const MergeLaunch& m, cudaStream_t stream) {
  const size_t state = merge_state_words(m.G, m.W) * 4;
  MergeLaunch l = m;
  l.state_in_smem = state <= kMergeSmemState ? 1 : 0;
  const size_t smem = l.state_in_smem ? state : 0;
  if (smem > 48 * 1024) {
    const cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(tail_merge_kernel), kMergeSmemState);
    if (e != cudaSuccess) return static_cast<int>(e);
  }
  tail_merge_kernel<<<m.BH, kMergeThreads, smem, stream>>>(l);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return static_cast<int>(e);
  merge_items_kernel<<<m.BH, kMergeThreads, 0, stream>>>(l);
  e = cudaGetLastError();
  if (e != cudaSuccess) return static_cast<int>(e);
  e = ensure_smem_attr(reinterpret_cast<const void*>(merge_balance_kernel), static_cast<int>(kBalanceSmem));
  if (e != cudaSuccess) return static_cast<int>(e);
  merge_balance_kernel<<<1, kBalanceThreads, kBalanceSmem, stream>>>(l);
  return static_cast<int>(cudaGetLastError());
}

}  // namespace isa_impl
