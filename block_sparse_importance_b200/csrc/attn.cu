// Sparse (and dense) flash attention over a block plan on sm_100a.
//
// "AB-Attention: Accurate Block Attention for Accelerating Video Diffusion
// Transformers" -- the discussion of the logit-shift form of the weights
// (each selected block's log(1/pi) is added to its scores before the softmax
// and the usual attention accumulation follows; only selected blocks receive
// exact attention) and of fine-grained selection with tiled execution (key /
// value blocks much smaller than a tile are gathered into full tensor-core
// tiles).
//
// Kernel design (one persistent CTA per SM, 18 warps):
//   * a work item is one query tile of <= 128 rows of one (batch, head,
//     group); a CTA takes items in pairs (A, B) and ping-pongs them so the
//     softmax of one tile overlaps the tensor-core work of the other;
//   * warp 16 (producer) streams K and V tiles of 128 rows through a 4-stage
//     shared-memory ring with TMA, gathering every plan block of k_block rows
//     (16..128) into its place in the tile (one box per block and 64-column
//     chunk, 128-byte swizzle, out-of-range rows zero-filled);
//   * warp 17 (MMA) runs converged and issues tcgen05.mma through an elected
//     lane: S = Q K^T into TMEM (both operands K-major in shared memory),
//     then O += P V with P read from TMEM and V MN-major in shared memory,
//     fp32 accumulation in TMEM;
//   * warps 0-7 / 8-15 (softmax of tile A / B): two warps per 32-row TMEM
//     lane slice, each over one 64-column half of the row.  They read S, add
//     scale*s + log_w(block) (log2 units), mask invalid rows, agree on the
//     row max through shared memory, keep an online max that is raised (and
//     their half of O rescaled in TMEM) only when it grows by more than 2^8,
//     write P = exp2(z - max) as bf16 over S's columns, and finally normalise
//     their half of O and store bf16 rows and the log-sum-exp.
// When both tiles of a pair read the same plan (dense mode, or two tiles of
// one cluster) the K/V stream is loaded once and used by both.
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

struct __align__(16) TileDesc {
  int g, row0, nrows, pad;
};

struct AttnArgs {
  int BH, N, G, S, Bk, nK, q_block, mode;
  int bk_shift;  // log2(Bk): plan positions are split into block and offset by shifts
  int tiles_per_head;  // groups / dense modes
  int T;               // KV tiles per query tile
  const int32_t* idx;
  const float* log_w;
  __nv_bfloat16* out;
  float* lse;
  const TileDesc* tiles;  // list mode
  const int* tile_count;  // list mode
  float scale_log2;
  int* status;
  uint64_t timeout;  // per-wait limit, ns
  int stall;         // test hook (failure detection)
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
};

// max of 16 consecutive fp32 values held as raw bits, by 3-input max
__device__ __forceinline__ float max16(const uint32_t* v) {
  auto f = [&](int i) { return __uint_as_float(v[i]); };
  const float m0 = fmax3f(f(0), f(1), f(2)), m1 = fmax3f(f(3), f(4), f(5)), m2 = fmax3f(f(6), f(7), f(8));
  const float m3 = fmax3f(f(9), f(10), f(11)), m4 = fmax3f(f(12), f(13), f(14));
  return fmaxf(fmax3f(m0, m1, m2), fmax3f(m3, m4, f(15)));
}

__device__ __forceinline__ bool decode_work(const AttnArgs& a, int tph, int n_work, int w, Work& r) {
  if (w >= n_work) return false;
  r.bh = w / tph;
  const int t = w - r.bh * tph;
  if (a.mode == kAttnDense) {
    r.g = 0;
    r.row0 = t * kTileRows;
    r.nrows = min(kTileRows, a.N - r.row0);
  } else if (a.mode == kAttnGroups) {
    r.g = t;
    r.row0 = t * a.q_block;
    r.nrows = min(a.q_block, a.N - r.row0);
  } else {
    const TileDesc td = a.tiles[t];
    r.g = td.g;
    r.row0 = td.row0;
    r.nrows = td.nrows;
  }
  return r.nrows > 0;
}

// The MMA issue order of one pair; the producer walks the same list to load
// the ring in consumption order.  f(kind, side, j): kind 0 = S = Q K_j^T,
// kind 1 = O += P V_j.  Returns false to stop early.
template <typename F>
__device__ __forceinline__ bool for_each_op(bool pa, bool pb, int T, F&& f) {
  if (pa && !f(0, 0, 0)) return false;
  if (pb && !f(0, 1, 0)) return false;
  for (int j = 0; j < T; ++j) {
    if (pa) {
      if (!f(1, 0, j)) return false;
      if (j + 1 < T && !f(0, 0, j + 1)) return false;
    }
    if (pb) {
      if (!f(1, 1, j)) return false;
      if (j + 1 < T && !f(0, 1, j + 1)) return false;
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

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const AttnArgs a) {
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

  const int tph = (a.mode == kAttnList) ? *a.tile_count : a.tiles_per_head;
  const int n_work = a.BH * tph;
  const int n_pairs = (n_work + 1) >> 1;
  const int T = a.T;
  const bool dense = a.mode == kAttnDense;
  const int bpt = dense ? 1 : kTileRows >> a.bk_shift;  // plan blocks per KV tile

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    uint32_t ring_pos = 0, q_loads0 = 0, q_loads1 = 0;
    bool ok = true;
    for (int p = blockIdx.x; p < n_pairs && ok; p += gridDim.x) {
      Work wk[2];
      const bool pr0 = decode_work(a, tph, n_work, 2 * p, wk[0]);
      const bool pr1 = decode_work(a, tph, n_work, 2 * p + 1, wk[1]);
      const bool shared = pr0 && pr1 && wk[0].bh == wk[1].bh && (dense || wk[0].g == wk[1].g);
      for (int x = 0; x < 2 && ok; ++x) {
        const bool present = x == 0 ? pr0 : pr1;
        if (!present) continue;
        uint32_t& q_loads = x ? q_loads1 : q_loads0;
        const Work& wx = x ? wk[1] : wk[0];
        if (lane == 0) ok = mbar_wait(bar(L::kBarQEmpty + x), (q_loads & 1u) ^ 1u, abort_flag, a.timeout);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        ++q_loads;
        if (lane == 0) {
          mbar_arrive_expect_tx(bar(L::kBarQFull + x), L::kQBytes);
          const uint32_t dst = base + L::kQOff + x * L::kQBytes;
#pragma unroll
          for (int c = 0; c < D / 64; ++c)
            tma_load_3d(dst + c * L::kChunkBytes, &tm_q, bar(L::kBarQFull + x), c * 64, wx.row0, wx.bh);
        }
      }
      if (!ok) break;
      ok = for_each_op(pr0, pr1, T, [&](int kind, int side, int j) -> bool {
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
        if (dense) {
          if (lane == 0) {
#pragma unroll
            for (int c = 0; c < D / 64; ++c)
              tma_load_3d(dst + c * L::kChunkBytes, map, bar(L::kBarKVFull + slot), c * 64, j * kTileRows, w.bh);
          }
        } else if (lane < bpt) {
          const int s = j * bpt + lane;
          int y = a.N;  // past the end: the box is zero-filled and masked
          if (s < a.S) {
            const int b = a.idx[(static_cast<int64_t>(w.bh) * a.G + w.g) * a.S + s];
            if (b >= 0 && b < a.nK) {
              y = b * a.Bk;
            } else {
              *bad_index = 1;
            }
          }
#pragma unroll
          for (int c = 0; c < D / 64; ++c)
            tma_load_3d(dst + c * L::kChunkBytes + lane * a.Bk * 128, map, bar(L::kBarKVFull + slot), c * 64, y,
                        w.bh);
        }
        ++ring_pos;  // counts only items whose copies were issued
        return true;
      });
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
        const bool pr0 = decode_work(a, tph, n_work, 2 * p, wk[0]);
        const bool pr1 = decode_work(a, tph, n_work, 2 * p + 1, wk[1]);
        const bool shared = pr0 && pr1 && wk[0].bh == wk[1].bh && (dense || wk[0].g == wk[1].g);
        ok = for_each_op(pr0, pr1, T, [&](int kind, int side, int j) -> bool {
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
              if (j == T - 1) tc_commit(bar(L::kBarQEmpty + side));
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
            if (j == T - 1 && elect_one()) tc_commit(bar(L::kBarODone + side));
          }
          if (release && elect_one()) tc_commit(bar(L::kBarKVEmpty + slot));
          return true;
        });
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
      if (!decode_work(a, tph, n_work, 2 * p + x, w)) continue;
      const int64_t prow = (static_cast<int64_t>(w.bh) * a.G + w.g) * a.S;
      float m_used = 0.0f, l_sum = 0.0f;
      // per 16-column chunk of this half: log-weight (log2 units) and number of
      // valid key rows; lanes 0..3 each work out one chunk.  The plan's entries
      // for tile j+1 are loaded while tile j runs and decoded a tile later.
      auto fetch = [&](int jj, int& rb, float& rlw) {
        rb = -1;
        rlw = 0.0f;
        if (!dense && lane < 4) {
          const int s = (jj * kTileRows + 64 * hf + lane * 16) >> a.bk_shift;
          if (s < a.S) {
            rb = a.idx[prow + s];
            rlw = a.log_w[prow + s];
          }
        }
      };
      auto decode = [&](int jj, int rb, float rlw, float& bias_o, int& valid_o) {
        bias_o = 0.0f;
        valid_o = 0;
        if (lane < 4) {
          const int pos = jj * kTileRows + 64 * hf + lane * 16;
          if (dense) {
            valid_o = max(0, min(16, a.N - pos));
          } else if (rb >= 0 && rb < a.nK) {
            const int within = pos & (a.Bk - 1);
            valid_o = max(0, min(16, min(a.Bk, a.N - rb * a.Bk) - within));
            bias_o = rlw * kLog2e;
          }
        }
      };
      int nb_idx;
      float nb_lw;
      fetch(0, nb_idx, nb_lw);
      for (int j = 0; j < T; ++j) {
        const int cur_idx = nb_idx;
        const float cur_lw = nb_lw;
        if (j + 1 < T) fetch(j + 1, nb_idx, nb_lw);
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
        if (j == 0) {
          m_used = mx == -INFINITY ? 0.0f : mx;
        } else if (__any_sync(0xffffffffu, mx > m_used + kRescaleLog2)) {
          // raise the running max and rescale this half's O columns and sum
          const float m_new = fmaxf(m_used, mx);
          const float f = fast_exp2(m_used - m_new);
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
      const bool valid = row < w.nrows;
      const int64_t grow = static_cast<int64_t>(w.bh) * a.N + w.row0 + row;
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

// Builds the query-tile list of the list mode: cluster (or group) g of rows
// [off[g], off[g+1]) contributes ceil(n_g / 128) tiles.  Validates offsets.
__global__ void build_tile_list(const int32_t* off, int G, int N, int q_block, TileDesc* tiles, int* count,
                                int* status) {
  __shared__ int s_tot[1024];
  __shared__ int s_bad;
  const int t = threadIdx.x, nt = blockDim.x;
  if (t == 0) s_bad = 0;
  __syncthreads();
  auto lo_of = [&](int g) { return off ? off[g] : min(g * q_block, N); };
  const int per = (G + nt - 1) / nt;
  const int g0 = min(G, t * per), g1 = min(G, g0 + per);
  int n = 0;
  for (int g = g0; g < g1; ++g) {
    const int lo = lo_of(g), hi = lo_of(g + 1);
    if (hi <= lo || lo < 0 || hi > N) s_bad = 1;
    n += (max(hi - lo, 0) + kTileRows - 1) / kTileRows;
  }
  if (t == 0 && (lo_of(0) != 0 || lo_of(G) != N)) s_bad = 1;
  s_tot[t] = n;
  __syncthreads();
  for (int d = 1; d < nt; d <<= 1) {  // inclusive scan of per-thread tile counts
    const int v = t >= d ? s_tot[t - d] : 0;
    __syncthreads();
    s_tot[t] += v;
    __syncthreads();
  }
  if (s_bad) {
    if (t == 0) {
      *count = 0;
      atomicCAS(status, 0, kStatusDeviceCheck);
    }
    return;
  }
  int o = s_tot[t] - n;
  for (int g = g0; g < g1; ++g) {
    const int lo = lo_of(g), hi = lo_of(g + 1);
    for (int r = lo; r < hi; r += kTileRows) tiles[o++] = TileDesc{g, r, min(kTileRows, hi - r), 0};
  }
  if (t == nt - 1) *count = s_tot[t];
}

template <int D>
int launch_d(const AttnLaunch& l, const void* q, const void* k, const void* v, cudaStream_t stream) {
  using Lay = Layout<D>;
  const int BH = l.B * l.H;
  CUtensorMap tq, tk, tv;
  const int kv_rows = l.mode == kAttnDense ? kTileRows : l.Bk;
  if (!make_bf16_map(&tq, q, BH, l.N, D, kTileRows) || !make_bf16_map(&tk, k, BH, l.N, D, kv_rows) ||
      !make_bf16_map(&tv, v, BH, l.N, D, kv_rows))
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
  int tiles_upper;
  if (l.mode == kAttnDense) {
    a.tiles_per_head = (l.N + kTileRows - 1) / kTileRows;
    a.T = a.tiles_per_head;
    tiles_upper = a.tiles_per_head;
  } else {
    a.T = (l.S * l.Bk + kTileRows - 1) / kTileRows;
    if (l.mode == kAttnGroups) {
      a.tiles_per_head = l.G;
      tiles_upper = l.G;
    } else {
      a.tiles = static_cast<const TileDesc*>(l.workspace);
      tiles_upper = l.G + l.N / kTileRows + 1;
      a.tile_count = reinterpret_cast<const int*>(static_cast<const char*>(l.workspace) +
                                                  static_cast<size_t>(tiles_upper) * sizeof(TileDesc));
      build_tile_list<<<1, 1024, 0, stream>>>(l.q_offsets, l.G, l.N, l.q_block, const_cast<TileDesc*>(a.tiles),
                                              const_cast<int*>(a.tile_count), l.status);
      cudaError_t e = cudaGetLastError();
      if (e != cudaSuccess) return static_cast<int>(e);
    }
  }
  const long long pairs = (static_cast<long long>(BH) * tiles_upper + 1) / 2;
  const int grid = static_cast<int>(pairs < l.num_sms ? pairs : l.num_sms);
  {
    const cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(attn_kernel<D>), Lay::kAlloc);
    if (e != cudaSuccess) return static_cast<int>(e);
  }
  attn_kernel<D><<<grid, kThreads, Lay::kAlloc, stream>>>(tq, tk, tv, a);
  return static_cast<int>(cudaGetLastError());
}

}  // namespace

size_t attn_list_workspace_bytes(int N, int G) {
  const size_t tiles_upper = static_cast<size_t>(G) + N / kTileRows + 1;
  return tiles_upper * sizeof(TileDesc) + 16;
}

int launch_attention(const AttnLaunch& l, const void* q, const void* k, const void* v, cudaStream_t stream) {
  if (l.D == 128) return launch_d<128>(l, q, k, v, stream);
  if (l.D == 64) return launch_d<64>(l, q, k, v, stream);
  return -1;
}

}  // namespace isa_impl
