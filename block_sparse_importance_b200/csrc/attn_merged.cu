// Sparse flash attention over the tail-merged schedule of the permuted
// layout, on sm_100a.
//
// "iCATS: Fast Video Generation via Interaction-Aware Sparse Attention and
// Timestep-Adaptive Sparsity", AI summary, "Approach": the tail blocks of
// query clusters are merged with Hamming-nearest compatible clusters, to cut
// the padding of their last tiles.  The work items come from isa_tail_merge:
// every cluster's full 128-row tiles and single tails on the cluster's plan,
// and merged tiles whose members (one per 32-row quarter) share the union of
// their plans, each quarter on its own member's log-weights (-inf off its
// plan).
//
// The pipeline is the one of the tile-by-tile kernel (attn.cu): one persistent
// CTA per SM, 18 warps, tiles taken in pairs and ping-ponged, a TMA producer
// warp gathering K/V blocks through a 4-slot ring, one MMA warp issuing
// tcgen05.mma (S = Q K^T and O += P V in TMEM), 16 softmax warps in column
// halves.  What differs:
//   * a merged tile's Q rows are gathered per member in 8-row boxes into its
//     member's slot, and its K/V blocks come from the union list;
//   * the two tiles of a pair may run different numbers of KV tiles;
//   * a row that has met no block of its member's plan yet takes its first
//     finite max as it comes (up or down);
//   * the output rows of a merged tile go back to their members' rows.
// It is kept apart from attn.cu so that the tile-by-tile kernel's code is not
// touched by the merged mode's bookkeeping.
// Every barrier wait is bounded; on a timeout the CTA stops issuing work,
// drains what is in flight, frees its tensor memory and records
// ISA_ERR_TIMEOUT in the status word.

#include <cuda_bf16.h>

#include "isa_internal.h"
#include "ptx.cuh"
#include "tmap.h"

namespace isa_impl {
namespace {

using namespace isa_dev;

constexpr int kTileRows = 128;
constexpr int kRing = 4;
// 18 warps: 0-7 softmax of tile A and 8-15 of tile B (in each, warps 0-3
// take S columns 0-63 and warps 4-7 columns 64-127 of the same 128 rows),
// 16 TMA producer, 17 MMA issue.
constexpr int kThreads = 576;
constexpr int kProducerWarp = 16;
constexpr int kMmaWarp = 17;
constexpr uint32_t kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleLog2 = 8.0f;

struct AttnArgs {
  int BH, N, G, S, Bk, nK, q_block, mode;
  int bk_shift;  // log2(Bk): plan positions are split into block and offset by shifts
  int T;  // KV tiles of a query tile on its own plan
  const int32_t* idx;
  const float* log_w;
  __nv_bfloat16* out;
  float* lse;
  float scale_log2;
  int* status;
  uint64_t timeout;  // per-wait limit, ns
  int stall;         // test hook (failure detection)
  // merged mode: work items, merged tail tiles and their union lists and
  // log-weight tables (per (b, h) strides: G tiles, G S union entries,
  // 4 G S table entries); cluster offsets for the members' rows
  const WorkItem* items;
  const int* item_count;
  const MergeBin* bins;
  const int32_t* unions;
  const float* tables;
  const int32_t* q_offsets;
};

template <int D>
struct Layout {
  static constexpr uint32_t kQBytes = kTileRows * D * 2;
  static constexpr uint32_t kKVBytes = kTileRows * D * 2;
  static constexpr uint32_t kChunkBytes = kTileRows * 128;  // 128 rows x 64 bf16
  static constexpr uint32_t kQOff = 0;
  static constexpr uint32_t kRingOff = 2 * kQBytes;
  static constexpr uint32_t kBarOff = kRingOff + kRing * kKVBytes;
  static constexpr int kBarQFull = 0, kBarQEmpty = 2, kBarKVFull = 4, kBarKVEmpty = 4 + kRing,
                       kBarSFull = 4 + 2 * kRing, kBarPFull = kBarSFull + 2,
                       kBarODone = kBarPFull + 2, kBarFinal = kBarODone + 2, kBarStall = kBarFinal + 1,
                       kBarXchg = kBarStall + 1, kNumBars = kBarXchg + 8;
  static constexpr uint32_t kMiscOff = kBarOff + kNumBars * 8;
  // row max and row sum exchange between the two column halves:
  // [max | sum][tile][half][row]
  static constexpr uint32_t kXchgOff = kMiscOff + 16;
  static constexpr uint32_t kTotal = kXchgOff + 2 * 2 * 2 * 128 * 4;
  static constexpr uint32_t kAlloc = kTotal + 1024;
  // TMEM columns
  static constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO0 = 256, kColO1 = 256 + D;
};

struct Work {
  int bh, g, row0, nrows;
  int bin;  // merged mode: the head's merged tail tile, or -1
  int T;    // KV tiles of this query tile
};

// max of 16 consecutive fp32 values held as raw bits, by 3-input max
__device__ __forceinline__ float max16(const uint32_t* v) {
  auto f = [&](int i) { return __uint_as_float(v[i]); };
  const float m0 = fmax3f(f(0), f(1), f(2)), m1 = fmax3f(f(3), f(4), f(5)), m2 = fmax3f(f(6), f(7), f(8));
  const float m3 = fmax3f(f(9), f(10), f(11)), m4 = fmax3f(f(12), f(13), f(14));
  return fmaxf(fmax3f(m0, m1, m2), fmax3f(m3, m4, f(15)));
}

// Merged mode: item w of the work list.  A merged tail tile runs the union of
// its members' plans, ceil(ulen / bpt) KV tiles.
__device__ __forceinline__ bool decode_item(const AttnArgs& a, int n_work, int bpt, int w, Work& r) {
  if (w >= n_work) return false;
  const WorkItem it = a.items[w];
  r.bh = it.bh;
  r.g = it.g;
  r.row0 = it.row0;
  r.nrows = it.nrows;
  r.bin = -1;
  r.T = a.T;
  if (it.g < 0) {
    r.bin = -1 - it.g;
    r.T = (a.bins[static_cast<int64_t>(it.bh) * a.G + r.bin].ulen + bpt - 1) / bpt;
  }
  return r.nrows > 0;
}

// The MMA issue order of one pair of tiles of Ta and Tb KV tiles; the
// producer walks the same list to load the ring in consumption order.
// f(kind, side, j): kind 0 = S = Q K_j^T, kind 1 = O += P V_j.  Returns false
// to stop early.
template <typename F>
__device__ __forceinline__ bool for_each_op2(bool pa, bool pb, int Ta, int Tb, F&& f) {
  if (pa && !f(0, 0, 0)) return false;
  if (pb && !f(0, 1, 0)) return false;
  const int Tm = max(pa ? Ta : 0, pb ? Tb : 0);
  for (int j = 0; j < Tm; ++j) {
    if (pa && j < Ta) {
      if (!f(1, 0, j)) return false;
      if (j + 1 < Ta && !f(0, 0, j + 1)) return false;
    }
    if (pb && j < Tb) {
      if (!f(1, 1, j)) return false;
      if (j + 1 < Tb && !f(0, 1, j + 1)) return false;
    }
  }
  return true;
}

__device__ __forceinline__ void set_status(int* status, int code) { atomicCAS(status, 0, code); }

// Wait that ignores the abort flag, used only to drain in-flight copies.
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > 200000000ull) break;
  }
}

// tm_q: 128-row Q boxes (a cluster's tiles); tm_q8: 8-row Q boxes (the
// members' tails of a merged tile).
template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_merged_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_q8,
                const AttnArgs a) {
  using L = Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_addr(smem_raw);
  const uint32_t base = (raw_addr + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw_addr);
  const uint32_t bars = base + L::kBarOff;
  auto bar = [&](int i) -> uint32_t { return bars + 8u * static_cast<uint32_t>(i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);
  volatile int* bad_index = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 8);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(L::kBarQFull + i), 1);
      mbar_init(bar(L::kBarQEmpty + i), 1);
      mbar_init(bar(L::kBarSFull + i), 1);
      mbar_init(bar(L::kBarPFull + i), 8);  // one arrival per softmax warp of the tile
      mbar_init(bar(L::kBarODone + i), 1);
    }
    for (int i = 0; i < kRing; ++i) {
      mbar_init(bar(L::kBarKVFull + i), 1);
      mbar_init(bar(L::kBarKVEmpty + i), 1);
    }
    mbar_init(bar(L::kBarFinal), 1);
    mbar_init(bar(L::kBarStall), 1);  // never arrived at: only the failure-detection hook waits on it
    for (int i = 0; i < 8; ++i) mbar_init(bar(L::kBarXchg + i), 2);  // the two warps of a row slice
    *abort_flag = 0;
    *bad_index = 0;
    fence_mbar_init();
  }
  if (warp == kProducerWarp && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_addr(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int n_work = *a.item_count;
  const int n_pairs = (n_work + 1) >> 1;
  const int T = a.T;
  const int bpt = kTileRows >> a.bk_shift;  // plan blocks per KV tile
  auto decode = [&](int w, Work& r) -> bool { return decode_item(a, n_work, bpt, w, r); };

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    uint32_t ring_pos = 0, q_loads0 = 0, q_loads1 = 0;
    bool ok = true;
    for (int p = blockIdx.x; p < n_pairs && ok; p += gridDim.x) {
      Work wk[2];
      const bool pr0 = decode(2 * p, wk[0]);
      const bool pr1 = decode(2 * p + 1, wk[1]);
      const bool shared = pr0 && pr1 && wk[0].bh == wk[1].bh && wk[0].g == wk[1].g;
      for (int x = 0; x < 2 && ok; ++x) {
        const bool present = x == 0 ? pr0 : pr1;
        if (!present) continue;
        uint32_t& q_loads = x ? q_loads1 : q_loads0;
        const Work& wx = x ? wk[1] : wk[0];
        if (lane == 0) ok = mbar_wait(bar(L::kBarQEmpty + x), (q_loads & 1u) ^ 1u, abort_flag, a.timeout);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        ++q_loads;
        bool gathered = false;
        {
          if (wx.bin >= 0) {
            // a merged tile: each member's tail rows into its 8-row-aligned slot
            gathered = true;
            if (lane == 0) {
              const MergeBin& bn = a.bins[static_cast<int64_t>(wx.bh) * a.G + wx.bin];
              uint32_t boxes = 0;
              for (int m = 0; m < bn.n; ++m) {
                const int g = bn.g[m];
                boxes += static_cast<uint32_t>(((a.q_offsets[g + 1] - a.q_offsets[g]) % kTileRows + 7) / 8);
              }
              mbar_arrive_expect_tx(bar(L::kBarQFull + x), boxes * (D / 64) * 8u * 128u);
              const uint32_t dst = base + L::kQOff + x * L::kQBytes;
              for (int m = 0; m < bn.n; ++m) {
                const int g = bn.g[m];
                const int t = (a.q_offsets[g + 1] - a.q_offsets[g]) % kTileRows;
                const int r0 = a.q_offsets[g + 1] - t;
                for (int i = 0; i < (t + 7) / 8; ++i) {
#pragma unroll
                  for (int c = 0; c < D / 64; ++c)
                    tma_load_3d(dst + c * L::kChunkBytes + (bn.slot[m] + 8 * i) * 128, &tm_q8, bar(L::kBarQFull + x),
                                c * 64, r0 + 8 * i, wx.bh);
                }
              }
            }
          }
        }
        if (!gathered && lane == 0) {
          mbar_arrive_expect_tx(bar(L::kBarQFull + x), L::kQBytes);
          const uint32_t dst = base + L::kQOff + x * L::kQBytes;
#pragma unroll
          for (int c = 0; c < D / 64; ++c)
            tma_load_3d(dst + c * L::kChunkBytes, &tm_q, bar(L::kBarQFull + x), c * 64, wx.row0, wx.bh);
        }
      }
      if (!ok) break;
      // merged mode: where each side's KV blocks come from (its plan row, or a
      // merged tile's union list) and how many there are
      const int32_t* src0 = nullptr;
      const int32_t* src1 = nullptr;
      int len0 = 0, len1 = 0;
      {
        for (int x = 0; x < 2; ++x) {
          const Work& wx = x ? wk[1] : wk[0];
          const bool present = x ? pr1 : pr0;
          const int32_t* src = nullptr;
          int len = 0;
          if (present) {
            if (wx.bin >= 0) {
              const MergeBin& bn = a.bins[static_cast<int64_t>(wx.bh) * a.G + wx.bin];
              src = a.unions + static_cast<int64_t>(wx.bh) * a.G * a.S + bn.uoff;
              len = bn.ulen;
            } else {
              src = a.idx + (static_cast<int64_t>(wx.bh) * a.G + wx.g) * a.S;
              len = a.S;
            }
          }
          if (x) {
            src1 = src;
            len1 = len;
          } else {
            src0 = src;
            len0 = len;
          }
        }
      }
      auto op = [&](int kind, int side, int j) -> bool {
        if (shared && side == 1) return true;
        const Work& w = side ? wk[1] : wk[0];
        const uint32_t slot = ring_pos % kRing, use = ring_pos / kRing;
        bool good = true;
        if (lane == 0) good = mbar_wait(bar(L::kBarKVEmpty + slot), (use & 1u) ^ 1u, abort_flag, a.timeout);
        good = __shfl_sync(0xffffffffu, good, 0);
        if (!good) return false;
        if (lane == 0) mbar_arrive_expect_tx(bar(L::kBarKVFull + slot), L::kKVBytes);
        __syncwarp();
        const CUtensorMap* map = kind == 0 ? &tm_k : &tm_v;
        const uint32_t dst = base + L::kRingOff + slot * L::kKVBytes;
        if (lane < bpt) {
          const int s = j * bpt + lane;
          int y = a.N;  // past the end: the box is zero-filled and masked
          {
            const int32_t* src = side ? src1 : src0;
            const int len = side ? len1 : len0;
            if (s < len) {
              const int b = src[s];
              if (b >= 0 && b < a.nK) {
                y = b * a.Bk;
              } else {
                *bad_index = 1;
              }
            }
          }
#pragma unroll
          for (int c = 0; c < D / 64; ++c)
            tma_load_3d(dst + c * L::kChunkBytes + lane * a.Bk * 128, map, bar(L::kBarKVFull + slot), c * 64, y,
                        w.bh);
        }
        ++ring_pos;  // counts only items whose copies were issued
        return true;
      };
      ok = for_each_op2(pr0, pr1, wk[0].T, wk[1].T, op);
    }
    if ((!ok || *abort_flag) && lane == 0) {
      // drain the copies still in flight before the CTA may exit
      const uint32_t first = ring_pos > kRing ? ring_pos - kRing : 0;
      for (uint32_t i = first; i < ring_pos; ++i) drain_wait(bar(L::kBarKVFull + i % kRing), (i / kRing) & 1u);
      if (q_loads0) drain_wait(bar(L::kBarQFull + 0), (q_loads0 - 1) & 1u);
      if (q_loads1) drain_wait(bar(L::kBarQFull + 1), (q_loads1 - 1) & 1u);
    }
  } else if (warp == kMmaWarp) {
    // ----------------------------------------------------------------- MMA
    // The whole warp runs the loop and waits; one elected lane issues the
    // MMAs and commits.
    {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, 1);
      uint32_t ring_pos = 0, q_waits0 = 0, q_waits1 = 0, p_waits0 = 0, p_waits1 = 0;
      uint32_t last_k = 0, last_v = 0;
      // Shared-memory descriptors are built once: between the k-steps of one
      // operand only the start-address field (bits 0-13, address >> 4)
      // changes, and shared addresses stay below 2^18, so a constant add never
      // carries out of the field.  This keeps the issuing thread's work per
      // MMA to an add or two.
      const uint64_t desc_q0 = smem_desc_sw128(base + L::kQOff, 16, 1024);
      const uint64_t desc_q1 = smem_desc_sw128(base + L::kQOff + L::kQBytes, 16, 1024);
      const uint64_t desc_k = smem_desc_sw128(base + L::kRingOff, 16, 1024);
      const uint64_t desc_v = smem_desc_sw128(base + L::kRingOff, L::kChunkBytes, 1024);
      bool ok = true;
      if (a.stall) ok = mbar_wait_warp(bar(L::kBarStall), 0, abort_flag, a.timeout);
      for (int p = blockIdx.x; p < n_pairs && ok; p += gridDim.x) {
        Work wk[2];
        const bool pr0 = decode(2 * p, wk[0]);
        const bool pr1 = decode(2 * p + 1, wk[1]);
        const bool shared = pr0 && pr1 && wk[0].bh == wk[1].bh && wk[0].g == wk[1].g;
        auto op = [&](int kind, int side, int j) -> bool {
          int Ts = T;  // KV tiles of this side's query tile
          Ts = side ? wk[1].T : wk[0].T;
          const bool acquire = !(shared && side == 1);
          const bool release = !shared || side == 1;
          if (kind == 0 && j == 0) {
            uint32_t& qw = side ? q_waits1 : q_waits0;
            if (!mbar_wait_warp(bar(L::kBarQFull + side), qw & 1u, abort_flag, a.timeout)) return false;
            ++qw;
          }
          if (kind == 1) {
            uint32_t& pw = side ? p_waits1 : p_waits0;
            if (!mbar_wait_warp(bar(L::kBarPFull + side), pw & 1u, abort_flag, a.timeout)) return false;
            ++pw;
          }
          uint32_t slot;
          uint32_t& last = kind ? last_v : last_k;
          if (acquire) {
            slot = ring_pos % kRing;
            if (!mbar_wait_warp(bar(L::kBarKVFull + slot), (ring_pos / kRing) & 1u, abort_flag, a.timeout))
              return false;
            ++ring_pos;
            last = slot;
          } else {
            slot = last;
          }
          tc_fence_after();
          const uint64_t slot16 = (slot * L::kKVBytes) >> 4;
          if (kind == 0) {
            const uint64_t da = side ? desc_q1 : desc_q0;
            const uint64_t db = desc_k + slot16;
            const uint32_t d_s = tmem + (side ? L::kColS1 : L::kColS0);
#pragma unroll
            for (int k = 0; k < D / 16; ++k) {
              const uint64_t off16 = ((k >> 2) * L::kChunkBytes + (k & 3) * 32) >> 4;
              if (elect_one()) mma_ss(d_s, da + off16, db + off16, idesc_qk, k > 0 ? 1u : 0u);
            }
            if (elect_one()) {
              tc_commit(bar(L::kBarSFull + side));
              if (j == Ts - 1) tc_commit(bar(L::kBarQEmpty + side));
            }
          } else {
            const uint32_t a_p = tmem + (side ? L::kColS1 : L::kColS0);
            const uint32_t d_o = tmem + (side ? L::kColO1 : L::kColO0);
#pragma unroll
            for (int k = 0; k < kTileRows / 16; ++k) {
              // keys 0-63: P of the first column half at columns 0-31 of S;
              // keys 64-127: the second half's P at columns 64-95
              const uint32_t pcol = k < 4 ? 8 * k : 64 + 8 * (k - 4);
              if (elect_one())
                mma_ts(d_o, a_p + pcol, desc_v + slot16 + ((k * 2048) >> 4), idesc_pv, (j > 0 || k > 0) ? 1u : 0u);
            }
            if (j == Ts - 1 && elect_one()) tc_commit(bar(L::kBarODone + side));
          }
          if (release && elect_one()) tc_commit(bar(L::kBarKVEmpty + slot));
          return true;
        };
        ok = for_each_op2(pr0, pr1, wk[0].T, wk[1].T, op);
      }
      // every MMA must be complete before tensor memory is freed
      if (elect_one()) tc_commit(bar(L::kBarFinal));
      __syncwarp();
      drain_wait(bar(L::kBarFinal), 0);
    }
  } else if (warp < 16) {
    // ------------------------------------------------------------- softmax
    // one thread per (row, column half): row = TMEM lane, the half's 64
    // columns of S and D/2 columns of O
    const int x = warp >> 3;            // which tile of the pair
    const int hf = (warp >> 2) & 1;     // column half
    const int q4 = warp & 3;            // TMEM lane quarter
    const int row = q4 * 32 + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const uint32_t col_s = (x ? L::kColS1 : L::kColS0) + 64 * hf;  // this half's S; its P lands here too
    const uint32_t col_o = (x ? L::kColO1 : L::kColO0) + (D / 2) * hf;
    // separate max and sum slots: a half rewrites a slot only after its partner
    // has passed the read of the previous value (the next S needs the
    // partner's P, and the epilogue needs all of it)
    float* xchg_max = reinterpret_cast<float*>(smem + L::kXchgOff) + x * 256;        // [half][row]
    float* xchg_sum = reinterpret_cast<float*>(smem + L::kXchgOff) + 512 + x * 256;  // [half][row]
    const uint32_t xbar = bar(L::kBarXchg + x * 4 + q4);
    uint32_t s_waits = 0, o_waits = 0, x_waits = 0;
    bool ok = true;
    // combine a per-row value with the other half's (bounded wait on the pair's barrier)
    auto exchange = [&](float v, bool is_max, float& out) -> bool {
      float* xchg = is_max ? xchg_max : xchg_sum;
      xchg[hf * 128 + row] = v;
      __syncwarp();
      if (lane == 0) mbar_arrive(xbar);
      if (!mbar_wait_warp(xbar, x_waits & 1u, abort_flag, a.timeout)) return false;
      ++x_waits;
      const float o = xchg[(1 - hf) * 128 + row];
      out = is_max ? fmaxf(v, o) : v + o;
      return true;
    };
    for (int p = blockIdx.x; p < n_pairs && ok; p += gridDim.x) {
      Work w;
      if (!decode(2 * p + x, w)) continue;
      float m_used = 0.0f, l_sum = 0.0f;
      bool seen = true;  // the row has met a key of its plan (its row max is finite)
      // where this warp's blocks and log-weights come from: the cluster's plan
      // row, or a merged tile's union list and, since members take whole
      // 32-row quarters, the row of the table of this warp's member
      const int32_t* fidx;
      const float* flw;
      int flen;
      if (w.bin < 0) {
        const int64_t prow = (static_cast<int64_t>(w.bh) * a.G + w.g) * a.S;
        fidx = a.idx + prow;
        flw = a.log_w + prow;
        flen = a.S;
      } else {
        const MergeBin* bn = a.bins + static_cast<int64_t>(w.bh) * a.G + w.bin;
        int mw = 0;
        for (int m = 0; m < bn->n; ++m)
          if (q4 * 32 >= bn->slot[m]) mw = m;
        flen = bn->ulen;
        fidx = a.unions + static_cast<int64_t>(w.bh) * a.G * a.S + bn->uoff;
        flw = a.tables + static_cast<int64_t>(w.bh) * 4 * a.G * a.S + bn->toff + mw * flen;
      }
      // per 16-column chunk of this half: log-weight (log2 units) and number of
      // valid key rows; lanes 0..3 each work out one chunk.  The entries for
      // tile j+1 are loaded while tile j runs and decoded a tile later.
      auto fetch = [&](int jj, int& rb, float& rlw) {
        rb = -1;
        rlw = 0.0f;
        if (lane < 4) {
          const int s = (jj * kTileRows + 64 * hf + lane * 16) >> a.bk_shift;
          if (s < flen) {
            rb = fidx[s];
            rlw = flw[s];
          }
        }
      };
      auto decode = [&](int jj, int rb, float rlw, float& bias_o, int& valid_o) {
        bias_o = 0.0f;
        valid_o = 0;
        if (lane < 4) {
          const int pos = jj * kTileRows + 64 * hf + lane * 16;
          if (rb >= 0 && rb < a.nK) {
            const int within = pos & (a.Bk - 1);
            valid_o = max(0, min(16, min(a.Bk, a.N - rb * a.Bk) - within));
            bias_o = rlw * kLog2e;
          }
        }
      };
      int nb_idx;
      float nb_lw;
      fetch(0, nb_idx, nb_lw);
      for (int j = 0; j < w.T; ++j) {
        const int cur_idx = nb_idx;
        const float cur_lw = nb_lw;
        if (j + 1 < w.T) fetch(j + 1, nb_idx, nb_lw);
        float c_bias;
        int c_valid;
        decode(j, cur_idx, cur_lw, c_bias, c_valid);
        if (!mbar_wait_warp(bar(L::kBarSFull + x), s_waits & 1u, abort_flag, a.timeout)) {
          ok = false;
          break;
        }
        ++s_waits;
        tc_fence_after();
        // an empty chunk carries bias -inf; only a chunk cut by the end of the
        // sequence (a partial tail block) needs per-element masking
        if (c_valid == 0) c_bias = -INFINITY;
        const bool partial = __any_sync(0xffffffffu, c_valid > 0 && c_valid < 16);
        // pass 1: this half's row max of z = scale*s + log_w (log2 units);
        // scale > 0, so a chunk's max is scale * (max of s) + its bias
        float mx = -INFINITY;
        {
          uint32_t sv[2][16];
          tmem_ld16(lane_base + col_s, sv[0]);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            if (c < 3) tmem_ld16(lane_base + col_s + 16 * (c + 1), sv[(c + 1) & 1]);
            const uint32_t* v = sv[c & 1];
            const float bias = __shfl_sync(0xffffffffu, c_bias, c);
            float hm;
            if (!partial) {
              hm = max16(v);
            } else {
              const int nv = __shfl_sync(0xffffffffu, c_valid, c);
              hm = -INFINITY;
#pragma unroll
              for (int i = 0; i < 16; ++i)
                if (i < nv) hm = fmaxf(hm, __uint_as_float(v[i]));
            }
            mx = fmaxf(mx, fmaf(hm, a.scale_log2, bias));
            if (c < 3) tmem_wait_ld();
          }
        }
        if (!exchange(mx, true, mx)) {
          ok = false;
          break;
        }
        // merged tiles: a row that has met no key of its plan yet takes its
        // first finite max as it comes, up or down (mx is the row's, so both
        // halves decide alike)
        if (j == 0) {
          m_used = mx == -INFINITY ? 0.0f : mx;
          seen = mx != -INFINITY;
        } else if (__any_sync(0xffffffffu,
                              mx > m_used + kRescaleLog2 || (!seen && mx > -INFINITY))) {
          // raise the running max and rescale this half's O columns and sum
          const bool fresh = !seen && mx > -INFINITY;
          const float m_new = fresh ? mx : fmaxf(m_used, mx);
          const float f = fresh ? 0.0f : fast_exp2(m_used - m_new);
          seen = seen || fresh;
          m_used = m_new;
          l_sum *= f;
#pragma unroll
          for (int c = 0; c < D / 64; ++c) {
            uint32_t o[32];
            tmem_ld32(lane_base + col_o + 32 * c, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * f);
            tmem_st32(lane_base + col_o + 32 * c, o);
          }
          tmem_wait_st();
        }
        // pass 2: P = exp2(z - max) as bf16 pairs; chunk c's 8 packed columns
        // land on columns 8c.. of this half's S, which earlier chunks already read
        // (the scale-and-shift and the running sums use paired fp32 arithmetic:
        // one instruction for two elements)
        {
          uint64_t ls2[2] = {0ull, 0ull};  // (even, odd) partial sums; zero bits are (0.0f, 0.0f)
          const uint64_t sc2 = f2_pack(a.scale_log2, a.scale_log2);
          uint32_t sv[2][16];
          tmem_ld16(lane_base + col_s, sv[0]);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            if (c < 3) tmem_ld16(lane_base + col_s + 16 * (c + 1), sv[(c + 1) & 1]);
            const uint32_t* v = sv[c & 1];
            const float bm = __shfl_sync(0xffffffffu, c_bias, c) - m_used;
            const int nv = __shfl_sync(0xffffffffu, c_valid, c);
            const uint64_t bm2 = f2_pack(bm, bm);
            uint32_t pk[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              float x0, x1;
              f2_unpack(fma_f32x2(f2_pack(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1])), sc2, bm2), x0,
                        x1);
              if (partial) {
                x0 = 2 * i < nv ? x0 : -INFINITY;
                x1 = 2 * i + 1 < nv ? x1 : -INFINITY;
              }
              const float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
              ls2[i & 1] = add_f32x2(ls2[i & 1], f2_pack(p0, p1));
              pk[i] = pack_bf16x2(p0, p1);
            }
            tmem_st8(lane_base + col_s + 8 * c, pk);
            if (c < 3) tmem_wait_ld();
          }
          float s0, s1, s2, s3;
          f2_unpack(ls2[0], s0, s1);
          f2_unpack(ls2[1], s2, s3);
          l_sum += (s0 + s1) + (s2 + s3);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(L::kBarPFull + x));
      }
      if (!ok) break;
      if (!mbar_wait_warp(bar(L::kBarODone + x), o_waits & 1u, abort_flag, a.timeout)) {
        ok = false;
        break;
      }
      ++o_waits;
      tc_fence_after();
      float l_tot;
      if (!exchange(l_sum, false, l_tot)) {
        ok = false;
        break;
      }
      const float inv = l_tot > 0.0f ? 1.0f / l_tot : 0.0f;
      bool valid = row < w.nrows;
      int64_t grow = static_cast<int64_t>(w.bh) * a.N + w.row0 + row;
      {
        if (w.bin >= 0) {  // the row's member, and where its row goes
          const MergeBin* bn = a.bins + static_cast<int64_t>(w.bh) * a.G + w.bin;
          valid = false;
          for (int m = 0; m < bn->n; ++m) {
            const int g = bn->g[m];
            const int t = (a.q_offsets[g + 1] - a.q_offsets[g]) % kTileRows;
            if (row >= bn->slot[m] && row - bn->slot[m] < t) {
              valid = true;
              grow = static_cast<int64_t>(w.bh) * a.N + a.q_offsets[g + 1] - t + (row - bn->slot[m]);
            }
          }
        }
      }
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        uint32_t o[32];
        tmem_ld32(lane_base + col_o + 32 * c, o);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv, __uint_as_float(o[2 * i + 1]) * inv);
        if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(a.out + grow * D + (D / 2) * hf + 32 * c);
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
        }
      }
      if (valid && hf == 0 && a.lse) a.lse[grow] = (m_used + __log2f(l_tot)) * kLn2;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (tid == 0) {
    if (*abort_flag) set_status(a.status, kStatusTimeout);
    if (*bad_index) set_status(a.status, kStatusDeviceCheck);
  }
  if (warp == kMmaWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D>
int launch_merged_d(const AttnLaunch& l, const void* q, const void* k, const void* v, cudaStream_t stream) {
  using Lay = Layout<D>;
  const int BH = l.B * l.H;
  CUtensorMap tq, tk, tv, tq8;
  if (!make_bf16_map(&tq, q, BH, l.N, D, kTileRows) || !make_bf16_map(&tk, k, BH, l.N, D, l.Bk) ||
      !make_bf16_map(&tv, v, BH, l.N, D, l.Bk) || !make_bf16_map(&tq8, q, BH, l.N, D, 8))
    return -1;
  AttnArgs a{};
  a.BH = BH;
  a.N = l.N;
  a.G = l.G;
  a.S = l.S;
  a.Bk = l.Bk;
  a.bk_shift = 0;
  while ((1 << a.bk_shift) < l.Bk) ++a.bk_shift;
  a.nK = (l.N + l.Bk - 1) / l.Bk;
  a.q_block = l.q_block;
  a.mode = l.mode;
  a.idx = l.idx;
  a.log_w = l.log_w;
  a.out = static_cast<__nv_bfloat16*>(l.out);
  a.lse = l.lse;
  a.scale_log2 = l.scale * kLog2e;
  a.status = l.status;
  a.timeout = l.wait_timeout_ns ? l.wait_timeout_ns : kWaitTimeoutNs;
  a.stall = l.stall;
  a.T = (l.S * l.Bk + kTileRows - 1) / kTileRows;
  a.items = l.items;
  a.item_count = l.item_count;
  a.bins = l.bins;
  a.unions = l.unions;
  a.tables = l.tables;
  a.q_offsets = l.q_offsets;
  const long long pairs = (static_cast<long long>(BH) * (l.G + l.N / kTileRows) + 1) / 2;
  const int grid = static_cast<int>(pairs < l.num_sms ? pairs : l.num_sms);
  const cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(attn_merged_kernel<D>), Lay::kAlloc);
  if (e != cudaSuccess) return static_cast<int>(e);
  attn_merged_kernel<D><<<grid, kThreads, Lay::kAlloc, stream>>>(tq, tk, tv, tq8, a);
  return static_cast<int>(cudaGetLastError());
}

}  // namespace

int launch_attention_merged(const AttnLaunch& l, const void* q, const void* k, const void* v, cudaStream_t stream) {
  if (l.D == 128) return launch_merged_d<128>(l, q, k, v, stream);
  if (l.D == 64) return launch_merged_d<64>(l, q, k, v, stream);
  return -1;
}

}  // namespace isa_impl
