// Plan selection: exact set + SIP sample, one CTA per (batch, head, group).
//
// "AB-Attention: Accurate Block Attention for Accelerating Video Diffusion
// Transformers", discussion of Sampling with Inclusion-Probability weighting:
// the scores set inclusion probabilities, highly scored blocks may always
// enter, the sampler returns a fixed number of distinct blocks, and a block
// drawn with probability pi counts 1/pi times.  "InstaGen" abstract: the
// top-scoring blocks form an exact set, the rest is represented by a sample
// drawn in proportion to estimated attention.
//
// Everything that decides membership is integer arithmetic, so the plan is
// reproducible bit for bit:
//   * exact set: radix select (4 x 8-bit passes) on the fp32 bit patterns of
//     the mass (monotone for non-negative values), ties to the lower block;
//   * weights of the rest: w = floor(m / m_max * 2^31) + 1 in IEEE fp64;
//   * capping at pi = 1: repeat { T = sum of uncapped w, n' = n_s - #capped,
//     cap every block with n' w >= T } until stable (exact 64-bit sums);
//   * systematic PPS over the uncapped blocks in ascending order with one
//     uniform U = hi32(Philox4x64-10(key (seed,0), counter (g,h,b,0))[0]):
//     with q = floor(x n' / T) and r = x n' mod T, the number of points
//     (i + U 2^-32) T / n' below x is q + [r 2^32 > U T]; block j is drawn
//     when that count steps between W_{j-1} and W_j;
//   * drawn blocks get log_w = ln T - ln(n' w) (fp64, stored fp32).
// Rows of up to 2048 blocks go to a warp-per-row kernel; longer rows to a
// CTA-per-row kernel.  Both produce identical plans.

#include <cstdint>

#include "isa_internal.h"
#include "mma_sync.cuh"
#include "ptx.cuh"

namespace isa_impl {
namespace {

constexpr int kSelThreads = 256;
constexpr int kSelWarps = kSelThreads / 32;

// Philox4x64-10 (Salmon et al., SC'11), written for the device.
__device__ __forceinline__ uint64_t philox_word0(uint64_t c0, uint64_t c1, uint64_t c2, uint64_t c3,
                                                 uint64_t k0, uint64_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint64_t lo0 = 0xD2E7470EE14C6C93ULL * c0, hi0 = __umul64hi(0xD2E7470EE14C6C93ULL, c0);
    const uint64_t lo1 = 0xCA5A826395121157ULL * c2, hi1 = __umul64hi(0xCA5A826395121157ULL, c2);
    const uint64_t n0 = hi1 ^ c1 ^ k0, n2 = hi0 ^ c3 ^ k1;
    c0 = n0;
    c1 = lo1;
    c2 = n2;
    c3 = lo0;
    k0 += 0x9E3779B97F4A7C15ULL;
    k1 += 0xBB67AE8584CAA73BULL;
  }
  return c0;
}

// w = floor(m / m_max * 2^31) + 1 for a block of the rest with mass bits
// `key` (0 for non-positive mass), where the quotient is the IEEE fp64
// division rounded to nearest.  With c31 = RN(2^31 / m_max) the product
// y = RN(m c31) is within 2^-21 of X = m 2^31 / m_max (X < 2^31, two
// roundings of at most 2^-53 each), and RN(m / m_max) 2^31 can only reach the
// next integer above X when X lies within 2^-23 of it.  So when y is more
// than 2^-20 away from every integer, floor(y) is the rule's value; otherwise
// (rare) the division itself decides.
__device__ __noinline__ uint32_t quant_weight_div(uint32_t key, double mmax) {
  return static_cast<uint32_t>(floor(static_cast<double>(__uint_as_float(key)) / mmax * 2147483648.0)) + 1u;
}
__device__ __forceinline__ uint32_t quant_weight(uint32_t key, double mmax, double c31) {
  if (!(mmax > 0.0) || key == 0u) return 1u;
  const double y = static_cast<double>(__uint_as_float(key)) * c31;
  const double fl = floor(y);
  const double fr = y - fl;  // exact: fl <= y < fl + 1
  if (fr > 0x1p-20 && fr < 1.0 - 0x1p-20) return static_cast<uint32_t>(fl) + 1u;
  return quant_weight_div(key, mmax);
}

// Drops from L2, without write-back, every whole 128-byte line of a mass row
// that has been read in full (lines shared with a neighbouring row stay).
__device__ __forceinline__ void discard_row_lines(const float* row, int nK, int t, int nt) {
  const uintptr_t s0 = reinterpret_cast<uintptr_t>(row), s1 = s0 + static_cast<uintptr_t>(nK) * 4;
  const uintptr_t l0 = (s0 + 127) & ~static_cast<uintptr_t>(127), l1 = s1 & ~static_cast<uintptr_t>(127);
  for (uintptr_t p = l0 + static_cast<uintptr_t>(t) * 128; p < l1; p += static_cast<uintptr_t>(nt) * 128)
    asm volatile("discard.global.L2 [%0], 128;" ::"l"(p) : "memory");
}

struct SelShared {
  uint64_t red64[kSelWarps];
  uint32_t red32[kSelWarps];
  uint32_t hist[256];
  uint32_t sel_bin, remaining;
  int bad;
};

__device__ __forceinline__ uint64_t block_sum_u64(uint64_t v, SelShared& sh) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if (lane == 0) sh.red64[w] = v;
  __syncthreads();
  uint64_t t = 0;
#pragma unroll
  for (int i = 0; i < kSelWarps; ++i) t += sh.red64[i];
  return t;
}

__device__ __forceinline__ uint32_t block_max_u32(uint32_t v, SelShared& sh) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
  __syncthreads();
  if (lane == 0) sh.red32[w] = v;
  __syncthreads();
  uint32_t t = 0;
#pragma unroll
  for (int i = 0; i < kSelWarps; ++i) t = max(t, sh.red32[i]);
  return t;
}

// Exclusive prefix sum over the block in thread order; returns the prefix of
// this thread and writes the block total to *total.
__device__ __forceinline__ uint64_t block_scan_u64(uint64_t v, SelShared& sh, uint64_t* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  uint64_t inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint64_t t = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += t;
  }
  __syncthreads();
  if (lane == 31) sh.red64[w] = inc;
  __syncthreads();
  uint64_t before = 0, all = 0;
#pragma unroll
  for (int i = 0; i < kSelWarps; ++i) {
    if (i < w) before += sh.red64[i];
    all += sh.red64[i];
  }
  *total = all;
  return before + inc - v;
}

// CTA-per-row variant for rows longer than the warp kernel takes.  Thread t
// owns the contiguous blocks [t E, (t+1) E) (E odd, so that the threads of a
// warp reach distinct shared-memory banks), so every pass over the row is
// thread-local and each scan is a local prefix plus one block-wide scan.
// flags: bit0 exact, bit1 capped (or taken whole), bit2 drawn
__global__ void __launch_bounds__(kSelThreads) select_kernel(SelectLaunch a) {
  extern __shared__ __align__(16) uint8_t sm[];
  __shared__ SelShared sh;
  const int nK = a.nK;
  // shared memory: the keys, replaced in place by the weights of the rest
  // once the exact set and the rest's maximum are known (nothing reads a key
  // after that); a flag byte per block; the list of the drawn weights
  uint32_t* key = reinterpret_cast<uint32_t*>(sm);
  uint32_t* wq = key;
  uint8_t* flag = reinterpret_cast<uint8_t*>(key + nK);
  uint32_t* wl = reinterpret_cast<uint32_t*>(sm + ((static_cast<size_t>(nK) * 5 + 15) & ~static_cast<size_t>(15)));
  const int tid = threadIdx.x;
  const int64_t row = blockIdx.x;
  const int g = static_cast<int>(row % a.G);
  const int h = static_cast<int>((row / a.G) % a.H);
  const int b = static_cast<int>(row / (static_cast<int64_t>(a.G) * a.H));
  const float* m = a.mass + row * nK;
  const int S = a.n_exact + a.n_sample;
  // the row's split of the plan: fixed, or per row (top-p rule)
  const int n_exact = a.ne_rows ? min(max(a.ne_rows[row], 0), S) : a.n_exact;
  const int n_sample = S - n_exact;
  const int E = ((nK + kSelThreads - 1) / kSelThreads) | 1;
  const int i0 = min(nK, tid * E), i1 = min(nK, i0 + E);

  if (tid == 0) sh.bad = 0;
  for (int i = tid; i < 256; i += kSelThreads) sh.hist[i] = 0;
  __syncthreads();
  // the keys, with the first radix round's histogram of their top byte
  for (int i = tid; i < nK; i += kSelThreads) {
    const float v = m[i];
    uint32_t k = 0;
    if (!isfinite(v)) {
      sh.bad = 1;
    } else if (v > 0.0f) {
      k = __float_as_uint(v);
    }
    key[i] = k;
    flag[i] = 0;
    if (n_exact > 0) atomicAdd(&sh.hist[k >> 24], 1u);
  }
  __syncthreads();
  if (a.discard_mass) discard_row_lines(m, nK, tid, kSelThreads);

  // ---- exact set: the n_exact largest keys, ties to the lower index
  if (n_exact > 0) {
    uint32_t prefix = 0, mask = 0;
    if (tid == 0) sh.remaining = n_exact;
    for (int shift = 24; shift >= 0; shift -= 8) {
      if (shift < 24) {
        for (int i = tid; i < 256; i += kSelThreads) sh.hist[i] = 0;
        __syncthreads();
        for (int i = i0; i < i1; ++i) {
          const uint32_t k = key[i];
          if ((k & mask) == prefix) atomicAdd(&sh.hist[(k >> shift) & 255u], 1u);
        }
      }
      __syncthreads();
      if (tid < 32) {
        // lane l owns bins [8l, 8l+8); suffix sums from the top bin down
        uint32_t local = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) local += sh.hist[8 * tid + i];
        uint32_t suf = local;  // sum of bins owned by lanes >= tid
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t t = __shfl_down_sync(0xffffffffu, suf, o);
          if (tid + o < 32) suf += t;
        }
        const uint32_t need = sh.remaining;
        const uint32_t above = suf - local;  // bins of higher lanes
        const bool here = above < need && suf >= need;
        if (here) {
          uint32_t acc = above;
          for (int i = 7; i >= 0; --i) {
            const uint32_t c = sh.hist[8 * tid + i];
            if (acc + c >= need) {
              sh.sel_bin = 8 * tid + i;
              sh.remaining = need - acc;
              break;
            }
            acc += c;
          }
        }
      }
      __syncthreads();
      prefix |= sh.sel_bin << shift;
      mask |= 255u << shift;
      __syncthreads();
    }
    const uint32_t thr = prefix;
    const uint32_t take_ties = sh.remaining;
    uint64_t eq = 0;
    for (int i = i0; i < i1; ++i) eq += key[i] == thr ? 1u : 0u;
    uint64_t tot;
    uint64_t rank = block_scan_u64(eq, sh, &tot);
    for (int i = i0; i < i1; ++i) {
      const uint32_t k = key[i];
      const bool tie = k == thr;
      if (k > thr || (tie && rank < take_ties)) flag[i] = 1;
      rank += tie ? 1u : 0u;
    }
  }

  // ---- weights and capping over the rest (all per-block work is on the
  // thread's own segment; only the totals cross threads)
  const int n_rest = nK - n_exact;
  int n_left = 0;
  uint64_t T = 0;
  if (n_sample >= n_rest) {
    for (int i = i0; i < i1; ++i)
      if (!(flag[i] & 1)) flag[i] |= 2;
  } else if (n_sample > 0) {
    uint32_t kmax = 0;
    for (int i = i0; i < i1; ++i)
      if (!(flag[i] & 1)) kmax = max(kmax, key[i]);
    kmax = block_max_u32(kmax, sh);
    const double mmax = static_cast<double>(__uint_as_float(kmax));
    const double c31 = mmax > 0.0 ? 2147483648.0 / mmax : 0.0;
    // the weights with their sum and maximum in one pass
    uint64_t t0 = 0;
    uint32_t wmax = 0;
    for (int i = i0; i < i1; ++i) {
      const uint32_t w = (flag[i] & 1) ? 0u : quant_weight(key[i], mmax, c31);
      wq[i] = w;
      t0 += w;
      wmax = max(wmax, w);
    }
    T = block_sum_u64(t0, sh);
    n_left = n_sample;
    // capping (see the team kernel); no block is capped when even the largest
    // weight stays below T / n_s
    if (static_cast<uint64_t>(n_sample) * block_max_u32(wmax, sh) >= T) {
      int n_capped = 0;
      for (;;) {
        uint64_t add = 0;
        for (int i = i0; i < i1; ++i)
          if (!(flag[i] & 3) && static_cast<uint64_t>(n_left) * wq[i] >= T) ++add;
        add = block_sum_u64(add, sh);  // all counts are taken before any flag changes
        if (add == 0) break;
        for (int i = i0; i < i1; ++i)
          if (!(flag[i] & 3) && static_cast<uint64_t>(n_left) * wq[i] >= T) flag[i] |= 2;
        n_capped += static_cast<int>(add);
        uint64_t t = 0;
        for (int i = i0; i < i1; ++i)
          if (!(flag[i] & 3)) t += wq[i];
        T = block_sum_u64(t, sh);
        n_left = n_sample - n_capped;
      }
    }
    if (n_left > 0) {
      const uint32_t U = static_cast<uint32_t>(
          philox_word0(static_cast<uint32_t>(g), static_cast<uint32_t>(h + a.h_base), static_cast<uint32_t>(b + a.b_base), 0,
                       a.seed, 0) >>
          32);
      const uint64_t nl = static_cast<uint64_t>(n_left);
      const uint64_t ut_lo = static_cast<uint64_t>(U) * T;  // U T < 2^76
      const uint64_t ut_hi = __umul64hi(static_cast<uint64_t>(U), T);
      // points of the comb below x: q + [r 2^32 > U T] with q = floor(x n' / T)
      // and r = x n' - q T.  Walking x up by an uncapped weight (n' w < T)
      // moves r up by n' w and needs at most one reduction by T, so only the
      // start of each thread's segment takes a division.
      auto above = [&](uint64_t r_) -> bool {
        const uint64_t r_hi = r_ >> 32, r_lo = r_ << 32;
        return r_hi > ut_hi || (r_hi == ut_hi && r_lo > ut_lo);
      };
      uint64_t local = 0;
      for (int i = i0; i < i1; ++i)
        if (!(flag[i] & 3)) local += wq[i];
      uint64_t tot;
      const uint64_t xn0 = block_scan_u64(local, sh, &tot) * nl;
      uint64_t q = xn0 / T, r = xn0 - q * T;
      uint64_t f_prev = q + (above(r) ? 1u : 0u);
      for (int i = i0; i < i1; ++i) {
        if (!(flag[i] & 3)) {
          r += static_cast<uint64_t>(wq[i]) * nl;
          if (r >= T) {
            r -= T;
            ++q;
          }
          const uint64_t f = q + (above(r) ? 1u : 0u);
          if (f != f_prev) flag[i] |= 4;
          f_prev = f;
        }
      }
    }
  }

  // ---- write the plan row: exact ascending, then capped + drawn ascending.
  // The drawn blocks' log-weights are left to a second, converged pass over
  // the rest part of the row: per rest position, the drawn block's weight (0
  // for a capped block) goes to the list.
  int32_t* out_idx = a.idx + row * S;
  float* out_lw = a.log_w + row * S;
  const int n_rs = S - n_exact;
  uint64_t ne = 0, nr = 0;
  for (int i = i0; i < i1; ++i) {
    const uint8_t f = flag[i];
    ne += (f & 1) ? 1u : 0u;
    nr += (!(f & 1) && (f & 6)) ? 1u : 0u;
  }
  uint64_t tot;
  const uint64_t pre = block_scan_u64((ne << 32) | nr, sh, &tot);  // both counts < 2^32 (its barriers also
                                                                  // order every key read before the list)
  uint64_t pe = pre >> 32, pr = pre & 0xFFFFFFFFull;
  for (int i = i0; i < i1; ++i) {
    const uint8_t f = flag[i];
    if (f & 1) {
      if (pe < static_cast<uint64_t>(n_exact)) {
        out_idx[pe] = i;
        out_lw[pe] = 0.0f;
      }
      ++pe;
    } else if (f & 6) {
      if (pr < static_cast<uint64_t>(n_rs)) {
        out_idx[n_exact + pr] = i;
        wl[pr] = (f & 4) ? wq[i] : 0u;
      }
      ++pr;
    }
  }
  __syncthreads();
  const uint64_t tot_e = tot >> 32, tot_r = tot & 0xFFFFFFFFull;
  const double lnT = T > 0 ? log(static_cast<double>(T)) : 0.0;
  const int n_w = static_cast<int>(tot_r < static_cast<uint64_t>(n_rs) ? tot_r : static_cast<uint64_t>(n_rs));
  for (int k = tid; k < n_w; k += kSelThreads) {
    const uint32_t wv = wl[k];
    out_lw[n_exact + k] =
        wv ? static_cast<float>(lnT - log(static_cast<double>(static_cast<uint64_t>(n_left) * wv))) : 0.0f;
  }
  if (tid == 0) {
    if (sh.bad || tot_e != static_cast<uint64_t>(n_exact) || tot_e + tot_r != static_cast<uint64_t>(S))
      atomicCAS(a.status, 0, kStatusDeviceCheck);
  }
}

// ---------------------------------------------------------------------------
// Warp-per-row variant for rows of at most 32 * VPL blocks: lane l holds the
// contiguous blocks [l*VPL, (l+1)*VPL) in registers, so every scan is a local
// prefix plus one warp shuffle scan and no block-wide barrier is needed.  The
// exact set's threshold (the n_exact-th largest key, i.e. the largest t with
// #{key >= t} >= n_exact) comes from a 4-round radix select with a per-warp
// shared-memory histogram.  Same integer arithmetic and same results as
// select_kernel.
constexpr int kWarpRowsPerCta = 8;

// A team of W warps (32 W threads) selects one plan row.  Thread t holds the
// contiguous blocks [t VPL, (t+1) VPL) of the row in registers (VPL odd, so
// the threads' blocked reads of the staged row hit distinct banks); every
// cross-thread step is a warp shuffle plus, for W = 2, one exchange through
// shared memory behind the team's named barrier.
template <int W>
struct Team {
  uint64_t* red;    // W * 8 scratch words, used round-robin
  uint32_t bar_id;  // named barrier of the team (W = 2)
  int t, lane, wi;
  uint32_t slot;
  __device__ __forceinline__ void sync() const {
    if constexpr (W == 1)
      __syncwarp();
    else
      isa_dev::named_bar_sync(bar_id, 32 * W);
  }
  // the other warp's value of a warp-uniform quantity (W = 2)
  __device__ __forceinline__ uint64_t swap(uint64_t v) {
    uint64_t* r = red + (slot++ & 7u) * W;
    if (lane == 0) r[wi] = v;
    sync();
    return r[wi ^ 1];
  }
  __device__ __forceinline__ uint64_t sum_u64(uint64_t v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if constexpr (W == 1) return v;
    return v + swap(v);
  }
  __device__ __forceinline__ uint32_t sum_u32(uint32_t v) {
    v = __reduce_add_sync(0xffffffffu, v);
    if constexpr (W == 1) return v;
    return v + static_cast<uint32_t>(swap(v));
  }
  __device__ __forceinline__ uint32_t max_u32(uint32_t v) {
    v = __reduce_max_sync(0xffffffffu, v);
    if constexpr (W == 1) return v;
    return max(v, static_cast<uint32_t>(swap(v)));
  }
  // exclusive prefix over the team's threads in order
  __device__ __forceinline__ uint64_t excl_u64(uint64_t v) {
    uint64_t inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint64_t x = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += x;
    }
    if constexpr (W == 1) return inc - v;
    const uint64_t other = swap(__shfl_sync(0xffffffffu, inc, 31));
    return inc - v + (wi ? other : 0ull);
  }
};

// One plan row.  st: the row's mass as staged by the caller (element i at
// st[i]), reused for the log-weight list once the keys are in registers;
// hist: the team's 256-bin radix histogram; scr: VPL words of this thread's
// scratch (the drawn blocks' weights, in block order).  The passes over the
// thread's blocks are fused where the data allow: the first radix round with
// the key extraction, the exact set with the rest's maximum, the weights with
// their sum; the capping pass runs only when a weight can reach the cap.
template <int VPL, int W>
__device__ __forceinline__ void select_row_team(const SelectLaunch& a, const int64_t row, uint32_t* st,
                                                uint32_t* hist, uint32_t* scr, Team<W>& tm) {
  static_assert(VPL <= 64, "flags are 64-bit masks");
  constexpr int BPT = 256 / (32 * W);  // histogram bins owned by each thread
  const int nK = a.nK;
  const int t = tm.t, lane = tm.lane;
  const int g = static_cast<int>(row % a.G);
  const int h = static_cast<int>((row / a.G) % a.H);
  const int b = static_cast<int>(row / (static_cast<int64_t>(a.G) * a.H));
  const int base = t * VPL;
  const int nv = max(0, min(VPL, nK - base));  // blocks this thread holds
  const int S = a.n_exact + a.n_sample;
  // the row's split of the plan: fixed, or per row (top-p rule)
  const int n_exact = a.ne_rows ? min(max(a.ne_rows[row], 0), S) : a.n_exact;
  const int n_sample = S - n_exact;
  if (n_exact > 0) {
#pragma unroll
    for (int i = 0; i < BPT; ++i) hist[t * BPT + i] = 0u;
    tm.sync();
  }
  // ---- keys (mass bits; 0 for non-positive, non-finite or past the row),
  // with the first radix round's histogram of their top byte
  uint32_t key[VPL];
  bool bad = false;
#pragma unroll
  for (int v = 0; v < VPL; ++v) {
    uint32_t k = 0;
    if (v < nv) {
      const float x = __uint_as_float(st[base + v]);
      if (!isfinite(x)) {
        bad = true;
      } else if (x > 0.0f) {
        k = __float_as_uint(x);
      }
      if (n_exact > 0) atomicAdd(&hist[k >> 24], 1u);
    }
    key[v] = k;
  }
  // ---- exact set: the n_exact largest keys, ties to the lower block
  uint64_t ex = 0;    // bit v: block base+v is exact
  uint32_t kmax = 0;  // the largest key of the rest
  if (n_exact > 0) {
    // the n_exact-th largest key thr, by a radix select over the key bytes
    // from the top: a histogram of the keys that match the prefix so far, and
    // the bin holding the remaining rank (thread t owns bins BPT t ..
    // BPT t + BPT - 1, so the bins above a thread's are those of higher threads)
    uint32_t thr = 0, mask = 0, kk = static_cast<uint32_t>(n_exact);
#pragma unroll 1
    for (int shift = 24; shift >= 0; shift -= 8) {
      if (shift < 24) {
#pragma unroll
        for (int i = 0; i < BPT; ++i) hist[t * BPT + i] = 0u;
        tm.sync();
#pragma unroll
        for (int v = 0; v < VPL; ++v)
          if (v < nv && (key[v] & mask) == thr) atomicAdd(&hist[(key[v] >> shift) & 255u], 1u);
      }
      tm.sync();
      uint32_t cnt[BPT], local = 0;
#pragma unroll
      for (int i = 0; i < BPT; ++i) {
        cnt[i] = hist[t * BPT + i];
        local += cnt[i];
      }
      uint32_t suf = local;  // keys in the bins of threads >= this one (this warp)
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t x = __shfl_down_sync(0xffffffffu, suf, o);
        if (lane + o < 32) suf += x;
      }
      if constexpr (W == 2) {
        const uint32_t up = static_cast<uint32_t>(tm.swap(__shfl_sync(0xffffffffu, suf, 0)));
        if (tm.wi == 0) suf += up;  // the upper warp's bins are all above
      }
      const uint32_t above = suf - local;
      const bool here = above < kk && suf >= kk;
      uint32_t sel = 0, rem = 0;
      if (here) {
        uint32_t acc = above;
#pragma unroll
        for (int i = BPT - 1; i >= 0; --i) {
          if (rem == 0 && acc + cnt[i] >= kk) {
            sel = BPT * t + i;
            rem = kk - acc;
          }
          acc += cnt[i];
        }
      }
      // exactly one thread of the team holds the bin: share it
      uint64_t pick = here ? ((static_cast<uint64_t>(sel) << 32) | rem) : 0ull;
      const uint32_t src = __ballot_sync(0xffffffffu, here);
      pick = src ? __shfl_sync(0xffffffffu, pick, __ffs(src) - 1) : 0ull;
      if constexpr (W == 2) pick |= tm.swap(pick);  // the warp without it contributes 0
      sel = static_cast<uint32_t>(pick >> 32);
      rem = static_cast<uint32_t>(pick);
      thr |= sel << shift;
      mask |= 255u << shift;
      kk = rem;
      if constexpr (W == 1) tm.sync();  // every lane has read the histogram before it is cleared
    }
    // keys above thr are exact, and the lowest kk of the keys equal to thr
    // (kk = n_exact - #{key > thr}); the rest's maximum is thr if a tie is
    // left over, else the largest key below thr
    uint64_t eqm = 0;
    uint32_t below = 0;
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
      if (v < nv) {
        if (key[v] > thr) ex |= 1ull << v;
        if (key[v] == thr) eqm |= 1ull << v;
        if (key[v] < thr) below = max(below, key[v]);
      }
    }
    uint32_t rank = static_cast<uint32_t>(tm.excl_u64(__popcll(eqm)));
    bool tie_left = false;
    for (uint64_t m = eqm; m; m &= m - 1) {
      if (rank < kk)
        ex |= m & (~m + 1);
      else
        tie_left = true;
      ++rank;
    }
    kmax = tie_left ? thr : below;
  } else {
#pragma unroll
    for (int v = 0; v < VPL; ++v)
      if (v < nv) kmax = max(kmax, key[v]);
  }
  // ---- the rest: weights (in registers, in place of the keys), capping,
  // systematic PPS.  Every loop over the thread's blocks is unrolled, so the
  // per-block flags are bits at constant positions.
  const int n_rest = nK - n_exact;
  uint64_t cap = 0, drawn = 0;  // bit v: capped (or taken whole), drawn
  uint64_t T = 0;
  int n_left = 0;
  if (n_sample >= n_rest) {
#pragma unroll
    for (int v = 0; v < VPL; ++v)
      if (v < nv && !((ex >> v) & 1)) cap |= 1ull << v;
  } else if (n_sample > 0) {
    kmax = tm.max_u32(kmax);
    const double mmax = static_cast<double>(__uint_as_float(kmax));
    const double c31 = mmax > 0.0 ? 2147483648.0 / mmax : 0.0;
    // w = floor(m / m_max * 2^31) + 1 on the rest; 0 on the exact set and past
    // the row; with their sum and maximum
    uint64_t tl = 0;
    uint32_t wmax = 0;
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
      uint32_t wv = 0;
      if (v < nv && !((ex >> v) & 1)) wv = quant_weight(key[v], mmax, c31);
      key[v] = wv;
      tl += wv;
      wmax = max(wmax, wv);
    }
    T = tm.sum_u64(tl);
    n_left = n_sample;
    // capping: repeat {T = sum of uncapped w, n' = n_s - #capped, cap every
    // uncapped block with n' w >= T} until nothing changes; no block is capped
    // when even the largest weight stays below T / n_s
    if (static_cast<uint64_t>(n_sample) * tm.max_u32(wmax) >= T) {
      int n_capped = 0;
      for (;;) {
        uint32_t add = 0;
        uint64_t newcap = 0;
#pragma unroll
        for (int v = 0; v < VPL; ++v) {
          if (key[v] != 0 && !((cap >> v) & 1) && static_cast<uint64_t>(n_left) * key[v] >= T) {
            newcap |= 1ull << v;
            ++add;
          }
        }
        const uint32_t add_all = tm.sum_u32(add);
        if (add_all == 0) break;
        cap |= newcap;
        n_capped += static_cast<int>(add_all);
        tl = 0;
#pragma unroll
        for (int v = 0; v < VPL; ++v)
          if (!((cap >> v) & 1)) tl += key[v];
        T = tm.sum_u64(tl);
        n_left = n_sample - n_capped;
      }
    }
    if (n_left > 0) {
      const uint32_t U = static_cast<uint32_t>(
          philox_word0(static_cast<uint32_t>(g), static_cast<uint32_t>(h + a.h_base), static_cast<uint32_t>(b + a.b_base), 0,
                       a.seed, 0) >>
          32);
      const uint64_t nl = static_cast<uint64_t>(n_left);
      // points of the comb below x: q + [r 2^32 > U T] with q = floor(x n' / T)
      // and r = x n' - q T; r 2^32 > U T is r > floor(U T / 2^32) for whole r.
      // Walking x up by an uncapped weight (n' w < T) moves r up by n' w and
      // needs at most one reduction by T, so only the start of each thread's
      // segment takes a division.  A drawn block's weight goes to the
      // thread's scratch, in block order.
      const uint64_t thr = static_cast<uint64_t>(U) * (T >> 32) + ((static_cast<uint64_t>(U) * (T & 0xFFFFFFFFull)) >> 32);
      const uint64_t xn0 = tm.excl_u64(tl) * nl;
      uint64_t r = xn0 % T;
      uint32_t q = static_cast<uint32_t>(xn0 / T);  // at most n'
      uint32_t f_prev = q + (r > thr ? 1u : 0u);
      int nd = 0;
#pragma unroll
      for (int v = 0; v < VPL; ++v) {
        if (key[v] != 0 && !((cap >> v) & 1)) {
          r += static_cast<uint64_t>(key[v]) * nl;
          if (r >= T) {
            r -= T;
            ++q;
          }
          const uint32_t f = q + (r > thr ? 1u : 0u);
          if (f != f_prev) {
            drawn |= 1ull << v;
            scr[nd++] = key[v];
          }
          f_prev = f;
        }
      }
    }
  }
  // ---- write the plan row: exact ascending, then capped + drawn ascending.
  // Each thread walks only its set flag bits.  The drawn blocks' log-weights
  // are left to a second, converged pass over the rest part of the row: each
  // thread records, per rest position it fills, the drawn block's weight (0
  // for a capped block) in the team's staged row, which no longer holds
  // anything the team reads.
  int32_t* out_idx = a.idx + row * S;
  float* out_lw = a.log_w + row * S;
  const int n_rs = S - n_exact;
  const uint32_t ne = __popcll(ex), nr = __popcll(cap | drawn);
  const uint64_t pre = tm.excl_u64((static_cast<uint64_t>(ne) << 32) | nr);  // both counts < 2^32
  uint32_t pe = static_cast<uint32_t>(pre >> 32);
  uint32_t pr = static_cast<uint32_t>(pre);
  tm.sync();
  for (uint64_t m = ex; m; m &= m - 1, ++pe) {
    if (pe < static_cast<uint32_t>(n_exact)) {
      out_idx[pe] = base + __ffsll(static_cast<long long>(m)) - 1;
      out_lw[pe] = 0.0f;
    }
  }
  int jd = 0;
  for (uint64_t m = cap | drawn; m; m &= m - 1, ++pr) {
    const uint64_t bit = m & (~m + 1);
    const bool is_drawn = (drawn & bit) != 0;
    const uint32_t wv = is_drawn ? scr[jd] : 0u;
    jd += is_drawn ? 1 : 0;
    if (pr < static_cast<uint32_t>(n_rs)) {
      out_idx[n_exact + pr] = base + __ffsll(static_cast<long long>(m)) - 1;
      st[pr] = wv;
    }
  }
  const uint64_t tot = tm.sum_u64((static_cast<uint64_t>(ne) << 32) | nr);  // also orders the list writes
  const uint32_t tot_e = static_cast<uint32_t>(tot >> 32), tot_r = static_cast<uint32_t>(tot);
  const double lnT = T > 0 ? log(static_cast<double>(T)) : 0.0;
  const int n_w = min(static_cast<int>(tot_r), n_rs);
  for (int k = t; k < n_w; k += 32 * W) {
    const uint32_t wv = st[k];
    out_lw[n_exact + k] =
        wv ? static_cast<float>(lnT - log(static_cast<double>(static_cast<uint64_t>(n_left) * wv))) : 0.0f;
  }
  const uint32_t any_bad = tm.sum_u32(bad ? 1u : 0u);
  if (t == 0 && (any_bad || tot_e != static_cast<uint32_t>(n_exact) || tot_e + tot_r != static_cast<uint32_t>(S)))
    atomicCAS(a.status, 0, kStatusDeviceCheck);
}

__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}

// Persistent teams of two warps: team w of the grid takes rows w, w + W,
// w + 2W, ... (W = the grid's teams) and stages the next row's mass in its
// second shared buffer (cp.async) while it selects the current one.
constexpr int kTeamWarps = 2;
constexpr int kTeamsPerCta = kWarpRowsPerCta / kTeamWarps;

template <int VPL>
struct TeamLayout {
  static constexpr int kSlice = 32 * kTeamWarps * VPL;  // one staged row
  // two staged rows, the histogram, the reduction scratch, the threads' drawn-weight scratch
  static constexpr int kTeamWords = 2 * kSlice + 256 + 2 * 8 * kTeamWarps + kSlice;
  static constexpr size_t kBytes = static_cast<size_t>(kTeamsPerCta) * kTeamWords * 4;
};

template <int VPL>
__global__ void __launch_bounds__(32 * kWarpRowsPerCta, VPL <= 19 ? 3 : 1) select_team_kernel(SelectLaunch a) {
  using L = TeamLayout<VPL>;
  extern __shared__ __align__(16) uint8_t sm[];
  const int warp = threadIdx.x >> 5;
  const int team = warp / kTeamWarps;
  const int64_t rows = static_cast<int64_t>(a.B) * a.H * a.G;
  uint32_t* tw = reinterpret_cast<uint32_t*>(sm) + team * L::kTeamWords;
  uint32_t* st = tw;
  uint32_t* hist = tw + 2 * L::kSlice;
  uint32_t* scr = hist + 256 + 2 * 8 * kTeamWarps;
  Team<kTeamWarps> tm;
  tm.red = reinterpret_cast<uint64_t*>(hist + 256);
  tm.bar_id = 1u + static_cast<uint32_t>(team);
  tm.t = threadIdx.x - team * 32 * kTeamWarps;
  tm.lane = threadIdx.x & 31;
  tm.wi = warp % kTeamWarps;
  tm.slot = 0;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kTeamsPerCta;
  int64_t row = static_cast<int64_t>(blockIdx.x) * kTeamsPerCta + team;
  auto stage = [&](int64_t r, uint32_t* dst) {
    const float* m = a.mass + r * a.nK;
    for (int i = tm.t; i < a.nK; i += 32 * kTeamWarps) cp_async4(isa_dev::smem_addr(dst + i), m + i);
  };
  using isa_dev::cp_async_commit;
  using isa_dev::cp_async_wait_group;
  if (row < rows) stage(row, st);
  cp_async_commit();
  int buf = 0;
  for (; row < rows; row += stride) {
    if (row + stride < rows) stage(row + stride, st + (buf ^ 1) * L::kSlice);
    cp_async_commit();
    cp_async_wait_group<1>();  // this thread's copies of the current row have landed
    tm.sync();
    if (a.discard_mass) discard_row_lines(a.mass + row * a.nK, a.nK, tm.t, 32 * kTeamWarps);
    select_row_team<VPL, kTeamWarps>(a, row, st + buf * L::kSlice, hist, scr + tm.t * VPL, tm);
    tm.sync();  // the buffer is restaged only after every thread is done with it
    buf ^= 1;
  }
  cp_async_wait_group<0>();
}

// ---------------------------------------------------------------------------
// Exact-set size by a share of the mass (the top-p rule of "iCATS": sparsity
// set by the share p of attention mass kept), one CTA per plan row, thread t
// over the contiguous blocks [t E, (t+1) E).  In exact integers, as the plan:
//   q_b = floor(m_b / m_max * 2^31) in fp64 for m_b > 0 (0 otherwise),
//   target = ceil(p * sum q) in fp64 (the sum is below 2^45: exact),
//   k_e = min(S, smallest k whose k largest blocks, ties to the lower block,
//         sum to >= target).
// The largest key t with sum_{key >= t} q >= target is found byte by byte
// from the top (a radix search whose histogram sums q instead of counting);
// all blocks above t are in, and of the blocks at t (equal q) the lowest
// ceil((target - sum_{key > t} q) / q_t).
__global__ void __launch_bounds__(kSelThreads) top_p_count_kernel(const float* __restrict__ mass, int nK,
                                                                  double top_p, int S, int32_t* __restrict__ ne_rows,
                                                                  int* status) {
  extern __shared__ __align__(16) uint8_t sm[];
  __shared__ SelShared sh;
  // per bin, the sum of q over the keys in it, as two 32-bit words (64-bit
  // shared-memory atomics are much slower): the low word, and the number of
  // times it wrapped
  __shared__ uint32_t hq_lo[256], hq_hi[256];
  __shared__ uint64_t s_above;  // sum of q over the keys above the current bin
  uint32_t* key = reinterpret_cast<uint32_t*>(sm);
  uint32_t* q = key + nK;
  const int tid = threadIdx.x;
  const int64_t row = blockIdx.x;
  const float* m = mass + row * nK;
  const int E = ((nK + kSelThreads - 1) / kSelThreads) | 1;
  const int i0 = min(nK, tid * E), i1 = min(nK, i0 + E);
  if (tid == 0) sh.bad = 0;
  __syncthreads();
  for (int i = tid; i < nK; i += kSelThreads) {
    const float v = m[i];
    uint32_t k = 0;
    if (!isfinite(v)) {
      sh.bad = 1;
    } else if (v > 0.0f) {
      k = __float_as_uint(v);
    }
    key[i] = k;
  }
  __syncthreads();
  uint32_t kmax = 0;
  for (int i = i0; i < i1; ++i) kmax = max(kmax, key[i]);
  kmax = block_max_u32(kmax, sh);
  const double mmax = static_cast<double>(__uint_as_float(kmax));
  auto quant = [&](uint32_t k) -> uint32_t {
    return (k != 0u && mmax > 0.0)
               ? static_cast<uint32_t>(floor(static_cast<double>(__uint_as_float(k)) / mmax * 2147483648.0))
               : 0u;
  };
  uint64_t local = 0;
  for (int i = i0; i < i1; ++i) {
    const uint32_t w = quant(key[i]);
    q[i] = w;
    local += w;
  }
  const uint64_t total = block_sum_u64(local, sh);
  const uint64_t target = static_cast<uint64_t>(ceil(top_p * static_cast<double>(total)));
  int k_e = 0;
  if (target > 0) {
    // byte by byte: among the keys that match the bytes found so far, the
    // highest bin whose q-sum, with everything above it, reaches the target
    uint32_t t = 0, mask = 0;
    uint64_t above = 0;
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int i = tid; i < 256; i += kSelThreads) {
        hq_lo[i] = 0;
        hq_hi[i] = 0;
      }
      __syncthreads();
      {
        // a thread's neighbouring blocks often share a bin: their q are
        // summed locally and added once per run
        auto add = [&](uint32_t bin, uint64_t v) {
          const uint32_t lo = static_cast<uint32_t>(v);
          const uint32_t old = atomicAdd(&hq_lo[bin], lo);
          const uint32_t carry = (static_cast<uint32_t>(v >> 32)) + (old + lo < old ? 1u : 0u);
          if (carry) atomicAdd(&hq_hi[bin], carry);
        };
        uint32_t run_bin = 256;
        uint64_t run = 0;  // < E 2^31
        for (int i = i0; i < i1; ++i) {
          const uint32_t k = key[i], w = q[i];  // w < 2^31
          if ((k & mask) == t && w != 0u) {
            const uint32_t bin = (k >> shift) & 255u;
            if (bin != run_bin) {
              if (run_bin < 256) add(run_bin, run);
              run_bin = bin;
              run = 0;
            }
            run += w;
          }
        }
        if (run_bin < 256) add(run_bin, run);
      }
      auto hq = [&](int i) -> uint64_t { return (static_cast<uint64_t>(hq_hi[i]) << 32) | hq_lo[i]; };
      __syncthreads();
      if (tid < 32) {
        // lane l owns bins [8l, 8l+8); suffix sums from the top bin down
        uint64_t local = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) local += hq(8 * tid + i);
        uint64_t suf = local;  // sum of the bins owned by lanes >= tid
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint64_t x = __shfl_down_sync(0xffffffffu, suf, o);
          if (tid + o < 32) suf += x;
        }
        const uint64_t need = target - above;  // > 0
        const uint64_t higher = suf - local;   // bins of higher lanes
        if (higher < need && suf >= need) {
          uint64_t acc = higher;
          for (int i = 7; i >= 0; --i) {
            const uint64_t c = hq(8 * tid + i);
            if (acc + c >= need) {
              sh.sel_bin = 8 * tid + i;
              s_above = above + acc;
              break;
            }
            acc += c;
          }
        }
      }
      __syncthreads();
      t |= sh.sel_bin << shift;
      mask |= 255u << shift;
      above = s_above;
      __syncthreads();
    }
    uint64_t gt_sum = 0, gt_cnt = 0;
    for (int i = i0; i < i1; ++i) {
      if (key[i] > t) {
        gt_sum += q[i];
        ++gt_cnt;
      }
    }
    gt_sum = block_sum_u64(gt_sum, sh);
    gt_cnt = block_sum_u64(gt_cnt, sh);
    const uint64_t q_t = quant(t);
    const uint64_t need = target - gt_sum;  // > 0: t is the largest key that reaches the target
    const uint64_t at_t = q_t > 0 ? (need + q_t - 1) / q_t : 0;
    k_e = static_cast<int>(min(static_cast<uint64_t>(S), gt_cnt + at_t));
  }
  if (tid == 0) {
    ne_rows[row] = k_e;
    if (sh.bad) atomicCAS(status, 0, kStatusDeviceCheck);
  }
}

template <int VPL>
int launch_select_team(const SelectLaunch& s, cudaStream_t stream) {
  using L = TeamLayout<VPL>;
  const long long rows = static_cast<long long>(s.B) * s.H * s.G;
  const size_t smem = L::kBytes;
  if (smem > 48 * 1024) {
    cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(select_team_kernel<VPL>), static_cast<int>(smem));
    if (e != cudaSuccess) return static_cast<int>(e);
  }
  int per_sm = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, select_team_kernel<VPL>,
                                                                32 * kWarpRowsPerCta, smem);
  if (e != cudaSuccess) return static_cast<int>(e);
  if (per_sm < 1) return static_cast<int>(cudaErrorInvalidConfiguration);
  const long long want = (rows + kTeamsPerCta - 1) / kTeamsPerCta;
  const long long cap = static_cast<long long>(s.num_sms > 0 ? s.num_sms : 148) * per_sm;
  const unsigned grid = static_cast<unsigned>(want < cap ? want : cap);
  select_team_kernel<VPL><<<grid, 32 * kWarpRowsPerCta, smem, stream>>>(s);
  return static_cast<int>(cudaGetLastError());
}

}  // namespace

int launch_top_p_count(const float* mass, int rows, int nK, double top_p, int S, int32_t* ne_rows, int* status,
                       cudaStream_t stream) {
  const size_t smem = static_cast<size_t>(nK) * 8 + 16;
  if (smem > 48 * 1024) {
    cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(top_p_count_kernel), static_cast<int>(smem));
    if (e != cudaSuccess) return static_cast<int>(e);
  }
  top_p_count_kernel<<<static_cast<unsigned>(rows), kSelThreads, smem, stream>>>(mass, nK, top_p, S, ne_rows, status);
  return static_cast<int>(cudaGetLastError());
}

int launch_select(const SelectLaunch& s, cudaStream_t stream) {
  constexpr int TT = 32 * kTeamWarps;  // threads per team
  if (s.nK <= TT * 5) return launch_select_team<5>(s, stream);
  if (s.nK <= TT * 9) return launch_select_team<9>(s, stream);
  if (s.nK <= TT * 19) return launch_select_team<19>(s, stream);
  if (s.nK <= TT * 33) return launch_select_team<33>(s, stream);
  // keys (weights in place) and flags, then the list of the drawn weights
  const size_t smem = ((static_cast<size_t>(s.nK) * 5 + 15) & ~static_cast<size_t>(15)) +
                      static_cast<size_t>(s.n_exact + s.n_sample) * 4;
  if (smem > 48 * 1024) {
    cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(select_kernel), static_cast<int>(smem));
    if (e != cudaSuccess) return static_cast<int>(e);
  }
  const long long rows = static_cast<long long>(s.B) * s.H * s.G;
  select_kernel<<<static_cast<unsigned>(rows), kSelThreads, smem, stream>>>(s);
  return static_cast<int>(cudaGetLastError());
}

}  // namespace isa_impl
