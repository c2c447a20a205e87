// Top-k selection, register-resident variant (HISA write-up, section 01: keep
// the k highest-scoring entries; ties go to the lower index).
//
// One CTA per row, each thread holding EPT (8, 16 or 32, chosen per row from its
// length) consecutive scores of the row in registers as order-preserving uint32
// keys (blocked layout: thread t owns positions [t*EPT, (t+1)*EPT)).  A 12-bit
// radix pass (4096-bin shared histogram) finds the bin that holds the k-th
// largest key.  The keys of that bin are gathered into shared memory (normally
// a few hundred at most) and one warp resolves them alone: up to 32 by counting,
// for each, the candidates above and equal to it; more by radix passes (8, 8 and
// 4 bits); either gives the exact k-th key K* and how many keys equal to it are
// taken.  Rows where more keys share the bin run a 12-bit and an 8-bit pass
// over the registers.
// Because the layout is blocked, a thread's selected elements form one bit mask
// (keys above K*, plus the first equal ones); the ordered output needs a single
// block-wide exclusive scan of per-thread (greater-than, equal-to) counts, and
// every thread then writes the positions of its mask's bits in ascending order.
#pragma once
#include "common.cuh"
#include "topk.cuh"

namespace hyb {

constexpr int kRegEPT = 32;
constexpr int kSelBins = 4096;       // 12-bit digits
constexpr int kSelCand = 512;        // boundary-bin candidates resolved over shared memory
constexpr int kSelOut = 2048;        // outputs staged in shared memory for coalesced stores (k <= kSelOut)

template <int THREADS>
struct RegSelSmem {
  alignas(16) uint32_t hist[kSelBins];
  uint32_t cand_key[kSelCand];
  int outbuf[kSelOut];
  uint32_t warp_tot[THREADS / 32];
  uint32_t warp_off[THREADS / 32];
  uint32_t total;
  uint32_t prefix, remaining, kth, need;
  uint32_t bin_count, n_slots;   // population of the last found bin; candidate slot counter
};

// Exclusive prefix sum over the CTA of one value per thread; `total` receives the sum.
template <int THREADS>
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, RegSelSmem<THREADS>& sh, uint32_t& total) {
  constexpr int NW = THREADS / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t u = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += u;
  }
  if (lane == 31) sh.warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const uint32_t t = lane < NW ? sh.warp_tot[lane] : 0u;
    uint32_t ti = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t u = __shfl_up_sync(0xffffffffu, ti, o);
      if (lane >= o) ti += u;
    }
    if (lane < NW) sh.warp_off[lane] = ti - t;
    if (lane == 31) sh.total = ti;
  }
  __syncthreads();
  total = sh.total;
  return sh.warp_off[warp] + incl - v;
}

// Finds the digit d of NBINS bins (each thread owns NBINS / THREADS consecutive bins)
// with above(d) < remaining <= above(d) + hist[d]; sets prefix |= d << shift and
// remaining -= above(d).  A thread keeps the sums of its groups of four bins, so the
// owner of the digit re-reads a single group.
template <int THREADS, int NBINS>
__device__ __forceinline__ void find_digit(RegSelSmem<THREADS>& sh, int shift) {
  constexpr int kBpt = NBINS / THREADS;
  static_assert(kBpt >= 1 && NBINS % THREADS == 0, "whole bins per thread");
  constexpr int kGs = kBpt % 4 == 0 ? 4 : 1;   // bins per group
  constexpr int kNg = kBpt / kGs;
  const uint32_t* mine = sh.hist + threadIdx.x * kBpt;
  uint32_t gsum[kNg], tot = 0;
#pragma unroll
  for (int g = 0; g < kNg; ++g) {
    if constexpr (kGs == 4) {
      const uint4 q = reinterpret_cast<const uint4*>(mine)[g];
      gsum[g] = q.x + q.y + q.z + q.w;
    } else {
      gsum[g] = mine[g];
    }
    tot += gsum[g];
  }
  const uint32_t rem = sh.remaining;
  const uint32_t prefix = sh.prefix;
  uint32_t total;
  const uint32_t before = block_exclusive_scan<THREADS>(tot, sh, total);
  uint32_t above = total - before - tot;    // keys in bins above this thread's range
  if (above < rem && rem <= above + tot) {
    int gsel = 0;
    bool found = false;
#pragma unroll
    for (int g = kNg - 1; g >= 0; --g) {
      if (!found && above + gsum[g] >= rem) { found = true; gsel = g; }
      if (!found) above += gsum[g];
    }
    uint32_t v[kGs];
    if constexpr (kGs == 4) {
      const uint4 q = reinterpret_cast<const uint4*>(mine)[gsel];
      v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
    } else {
      v[0] = gsum[gsel];
    }
    int d = 0;
    uint32_t h = 0, nrem = 0;
    found = false;
#pragma unroll
    for (int e = kGs - 1; e >= 0; --e) {
      if (!found && above + v[e] >= rem) { found = true; d = e; h = v[e]; nrem = rem - above; }
      if (!found) above += v[e];
    }
    sh.prefix = prefix | ((uint32_t)(threadIdx.x * kBpt + gsel * kGs + d) << shift);
    sh.remaining = nrem;
    sh.bin_count = h;
  }
  __syncthreads();
}

// One warp finds the k-th key among the n boundary-bin candidates in shared
// memory (every candidate shares the `done_bits` high bits already fixed in
// sh.prefix; sh.remaining is the rank sought among them).  Up to 32 candidates:
// each lane counts the candidates above and equal to its own; more: radix
// passes of up to 8 bits over a 256-bin histogram of the warp's own.  Leaves
// prefix = K* and remaining = how many keys equal to K* are taken.
template <int THREADS>
__device__ __forceinline__ void resolve_candidates_warp(RegSelSmem<THREADS>& sh, uint32_t n, int done_bits) {
  const int lane = threadIdx.x & 31;
  uint32_t prefix = sh.prefix, rem = sh.remaining;
  if (n <= 32) {
    const uint32_t mine = (uint32_t)lane < n ? sh.cand_key[lane] : 0u;
    uint32_t gt = 0, eq = 0;
    for (uint32_t j = 0; j < n; ++j) {
      const uint32_t kj = __shfl_sync(0xffffffffu, mine, j);
      gt += kj > mine ? 1u : 0u;
      eq += kj == mine ? 1u : 0u;
    }
    const bool hit = (uint32_t)lane < n && gt < rem && rem <= gt + eq;
    const int src = __ffs(__ballot_sync(0xffffffffu, hit)) - 1;
    prefix = __shfl_sync(0xffffffffu, mine, src);
    rem -= __shfl_sync(0xffffffffu, gt, src);
  } else {
    uint32_t mask = done_bits ? ~0u << (32 - done_bits) : 0u;
    uint32_t* h = sh.hist;
#pragma unroll 1
    for (int low = 32 - done_bits; low > 0;) {
      const int nb = low < 8 ? low : 8, shift = low - nb;
      const uint32_t dmask = (1u << nb) - 1u;
      for (int i = lane; i < 256; i += 32) h[i] = 0u;
      __syncwarp();
      for (uint32_t c = lane; c < n; c += 32) {
        const uint32_t kc = sh.cand_key[c];
        if ((kc & mask) == prefix) atomicAdd(&h[(kc >> shift) & dmask], 1u);
      }
      __syncwarp();
      uint32_t v[8], tot = 0;   // lane l owns digits 8l .. 8l+7
#pragma unroll
      for (int e = 0; e < 8; ++e) { v[e] = h[lane * 8 + e]; tot += v[e]; }
      uint32_t incl = tot;      // keys in this lane's digits and above
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t u = __shfl_down_sync(0xffffffffu, incl, o);
        if (lane + o < 32) incl += u;
      }
      uint32_t above = incl - tot, d = 0, nrem = 0;
      const bool mine = above < rem && rem <= above + tot;
      if (mine) {
#pragma unroll
        for (int e = 7; e >= 0; --e) {
          if (above + v[e] >= rem) { d = lane * 8 + e; nrem = rem - above; break; }
          above += v[e];
        }
      }
      const int src = __ffs(__ballot_sync(0xffffffffu, mine)) - 1;
      d = __shfl_sync(0xffffffffu, d, src);
      nrem = __shfl_sync(0xffffffffu, nrem, src);
      prefix |= d << shift;
      rem = nrem;
      mask |= dmask << shift;
      low = shift;
      __syncwarp();
    }
  }
  if (lane == 0) { sh.prefix = prefix; sh.remaining = rem; }
}

// Zeroes the first `nbins` histogram bins (a multiple of 4).
template <int THREADS>
__device__ __forceinline__ void zero_hist(RegSelSmem<THREADS>& sh, int nbins) {
  for (int b = threadIdx.x; b < nbins / 4; b += THREADS) reinterpret_cast<uint4*>(sh.hist)[b] = make_uint4(0, 0, 0, 0);
}

template <int THREADS, int EPT, typename Map>
__device__ void select_row_reg(const float* __restrict__ scores, int n, int k, int k_out, int* __restrict__ out,
                               Map map, RegSelSmem<THREADS>& sh) {
  const int tid = threadIdx.x;
  if (n <= k) {
    for (int i = tid; i < k_out; i += THREADS) out[i] = i < n ? map(i) : -1;
    return;
  }
  for (int i = k + tid; i < k_out; i += THREADS) out[i] = -1;
  const int base = tid * EPT;
  const int cnt = n - base < 0 ? 0 : (n - base > EPT ? EPT : n - base);
  // the row's scores are loaded first; the histogram is cleared while they arrive
  float f[EPT];
  if (cnt == EPT && (reinterpret_cast<uintptr_t>(scores + base) & 15) == 0) {
#pragma unroll
    for (int e = 0; e < EPT; e += 4) {
      const float4 q = *reinterpret_cast<const float4*>(scores + base + e);
      f[e] = q.x; f[e + 1] = q.y; f[e + 2] = q.z; f[e + 3] = q.w;
    }
  } else {
#pragma unroll
    for (int e = 0; e < EPT; ++e) f[e] = e < cnt ? scores[base + e] : 0.f;
  }
  constexpr int kLastBins = 256 < THREADS ? THREADS : 256;   // 8-bit pass, at least one bin per thread
  // ---- pass 0: bits 31..20
  zero_hist<THREADS>(sh, kSelBins);
  if (tid == 0) { sh.prefix = 0; sh.remaining = (uint32_t)k; sh.n_slots = 0; }
  uint32_t key[EPT];
#pragma unroll
  for (int e = 0; e < EPT; ++e) key[e] = e < cnt ? score_key(f[e]) : 0u;
  __syncthreads();
#pragma unroll
  for (int e = 0; e < EPT; ++e)
    if (e < cnt) atomicAdd(&sh.hist[key[e] >> 20], 1u);
  __syncthreads();
  find_digit<THREADS, kSelBins>(sh, 20);
  const uint32_t prefix0 = sh.prefix;
  // ---- the boundary bin's keys (their number is the bin's count)
  const uint32_t n_cand = sh.bin_count;
  __syncthreads();   // every thread has read the histogram results before it is reused
  if (n_cand <= (uint32_t)kSelCand) {
    // few: gather them (in any order); one warp resolves the low 20 bits over them alone
    // slots reserved once per warp: a warp scan of the per-thread counts, one atomic
    const int lane = tid & 31;
    uint32_t mine = 0;
#pragma unroll
    for (int e = 0; e < EPT; ++e) mine += (e < cnt && (key[e] >> 20) == (prefix0 >> 20)) ? 1u : 0u;
    uint32_t incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t u = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += u;
    }
    uint32_t wbase = 0;
    if (lane == 31 && incl > 0) wbase = atomicAdd(&sh.n_slots, incl);
    uint32_t slot = __shfl_sync(0xffffffffu, wbase, 31) + incl - mine;
#pragma unroll
    for (int e = 0; e < EPT; ++e)
      if (e < cnt && (key[e] >> 20) == (prefix0 >> 20)) sh.cand_key[slot++] = key[e];
    __syncthreads();
    if (tid < 32) resolve_candidates_warp<THREADS>(sh, n_cand, 12);
    __syncthreads();
  } else {
    // many keys share the first digit: a 12-bit and an 8-bit pass over the registers
    zero_hist<THREADS>(sh, kSelBins);
    __syncthreads();
#pragma unroll
    for (int e = 0; e < EPT; ++e)
      if (e < cnt && (key[e] & 0xFFF00000u) == prefix0) atomicAdd(&sh.hist[(key[e] >> 8) & 0xFFFu], 1u);
    __syncthreads();
    find_digit<THREADS, kSelBins>(sh, 8);
    const uint32_t prefix1 = sh.prefix;
    zero_hist<THREADS>(sh, kLastBins);
    __syncthreads();
#pragma unroll
    for (int e = 0; e < EPT; ++e)
      if (e < cnt && (key[e] & 0xFFFFFF00u) == prefix1) atomicAdd(&sh.hist[key[e] & 0xFFu], 1u);
    __syncthreads();
    find_digit<THREADS, kLastBins>(sh, 0);
  }
  const uint32_t kth = sh.prefix, need = sh.remaining;
  // ---- ordered output: bit e of gtm / eqm marks element e above / equal to K*
  static_assert(EPT <= 32, "one mask word per thread");
  uint32_t gtm = 0, eqm = 0;
#pragma unroll
  for (int e = 0; e < EPT; ++e) {
    if (e < cnt) {
      gtm |= (key[e] > kth ? 1u : 0u) << e;
      eqm |= (key[e] == kth ? 1u : 0u) << e;
    }
  }
  const uint32_t n_gt = __popc(gtm), n_eq = __popc(eqm);
  uint32_t total;
  const uint32_t before = block_exclusive_scan<THREADS>((n_gt << 16) | n_eq, sh, total);
  const uint32_t gt_before = before >> 16, eq_before = before & 0xFFFFu;
  // the equal keys taken are the first `need` in position order
  const uint32_t take = eq_before >= need ? 0u : min(need - eq_before, n_eq);
  while ((uint32_t)__popc(eqm) > take) eqm &= ~(0x80000000u >> __clz(eqm));   // drop the highest
  uint32_t sel = gtm | eqm;
  // selected positions in ascending order: staged in shared memory when k fits,
  // then stored by consecutive threads
  const bool staged = k <= kSelOut;
  int* dst = staged ? sh.outbuf : out;
  uint32_t slot = gt_before + min(eq_before, need);
  while (sel) {
    const int e = __ffs(sel) - 1;
    dst[slot++] = map(base + e);
    sel &= sel - 1;
  }
  if (staged) {
    __syncthreads();
    for (int i = tid; i < k; i += THREADS) out[i] = sh.outbuf[i];
  }
}

// Runs select_row_reg with the smallest register block that holds n keys
// (n <= THREADS * kRegEPT).
template <int THREADS, typename Map>
__device__ __forceinline__ void select_row_reg_any(const float* __restrict__ scores, int n, int k, int k_out,
                                                   int* __restrict__ out, Map map, RegSelSmem<THREADS>& sh) {
  if (n <= THREADS * 8) select_row_reg<THREADS, 8>(scores, n, k, k_out, out, map, sh);
  else if (n <= THREADS * 16) select_row_reg<THREADS, 16>(scores, n, k, k_out, out, map, sh);
  else select_row_reg<THREADS, kRegEPT>(scores, n, k, k_out, out, map, sh);
}

// Rows longer than one register block (kSegKeys keys): exact two-level selection.
// Pass 1 keeps the k best of every segment of kSegKeys keys; the k best of the
// row are among those (the order -- score descending, index ascending -- is the
// same within a segment), so pass 2 selects the k best of the segment winners.
// The winners are laid out segment after segment, each in ascending order, so a
// candidate's position orders ties exactly as its entry index does.
constexpr int kSegKeys = 1024 * kRegEPT;

struct OffsetMap {
  int lo;
  __device__ __forceinline__ int operator()(int p) const { return lo + p; }
};
struct CandIdxMap {
  const int* idx;
  __device__ __forceinline__ int operator()(int p) const { return idx[p]; }
};

__device__ __forceinline__ int seg_len(int n, int s) {
  const int len = n - s * kSegKeys;
  return len < 0 ? 0 : (len > kSegKeys ? kSegKeys : len);
}

__global__ void __launch_bounds__(1024, 1)
select_flat_seg_kernel(const float* __restrict__ S, const int* __restrict__ q_pos, int* __restrict__ cidx,
                       float* __restrict__ cscore, int T_, int i0, int nq, int r, int nc, int k, int ldS, int nseg) {
  __shared__ RegSelSmem<1024> sh;
  const int m = blockIdx.x, s = blockIdx.y, b = blockIdx.z;
  const size_t row = (size_t)b * T_ + i0 + m;
  const int n = visible_entries(q_pos[row], r, nc);
  const int len = seg_len(n, s);
  if (len == 0) return;
  int off = 0;   // candidates of the segments before this one
  for (int u = 0; u < s; ++u) off += seg_len(n, u) < k ? seg_len(n, u) : k;
  const int kk = len < k ? len : k;
  const size_t crow = ((size_t)b * nq + m) * (size_t)nseg * k + off;
  const float* srow = S + ((size_t)b * nq + m) * ldS + (size_t)s * kSegKeys;
  select_row_reg_any<1024>(srow, len, kk, kk, cidx + crow, OffsetMap{s * kSegKeys}, sh);
  __syncthreads();
  for (int i = threadIdx.x; i < kk; i += 1024) cscore[crow + i] = srow[cidx[crow + i] - s * kSegKeys];
}

template <int THREADS>
__global__ void __launch_bounds__(THREADS, THREADS <= 256 ? 4 : 1)
select_flat_merge_kernel(const int* __restrict__ q_pos, const int* __restrict__ cidx, const float* __restrict__ cscore,
                         int* __restrict__ idx, int T_, int i0, int nq, int r, int nc, int k, int nseg) {
  __shared__ RegSelSmem<THREADS> sh;
  const int m = blockIdx.x, b = blockIdx.y;
  const size_t row = (size_t)b * T_ + i0 + m;
  const int n = visible_entries(q_pos[row], r, nc);
  int total = 0;
  for (int u = 0; u < nseg; ++u) total += seg_len(n, u) < k ? seg_len(n, u) : k;
  const size_t crow = ((size_t)b * nq + m) * (size_t)nseg * k;
  select_row_reg_any<THREADS>(cscore + crow, total, k, k, idx + row * k, CandIdxMap{cidx + crow}, sh);
}

// Flat rows: row (b, i) keeps the k best of its visible entries.  Rows are taken
// last first: in causal order they are the longest, so the launch ends on short rows.
template <int THREADS>
__global__ void __launch_bounds__(THREADS, THREADS <= 256 ? 4 : 1)
select_flat_reg_kernel(const float* __restrict__ S, const int* __restrict__ q_pos, int* __restrict__ idx, int T_,
                       int i0, int nq, int r, int nc, int k, int ldS) {
  __shared__ RegSelSmem<THREADS> sh;
  const int b = blockIdx.y, m = nq - 1 - (int)blockIdx.x;
  const size_t row = (size_t)b * T_ + i0 + m;
  const int n = visible_entries(q_pos[row], r, nc);
  select_row_reg_any<THREADS>(S + ((size_t)b * nq + m) * ldS, n, k, k, idx + row * k, IdentityMap{}, sh);
}

// HISA stage 1: the partial block (if any) is always kept; the best full blocks
// fill the other slots.  blk row: kept blocks ascending, then -1.
template <int THREADS>
__global__ void __launch_bounds__(THREADS, THREADS <= 256 ? 4 : 1)
select_blocks_reg_kernel(const float* __restrict__ SB, const int* __restrict__ q_pos, int* __restrict__ blk, int T_,
                         int i0, int nq, int r, int nc, int block, int top_m, int ldB) {
  __shared__ RegSelSmem<THREADS> sh;
  const int b = blockIdx.y, m = blockIdx.x;
  const size_t row = (size_t)b * T_ + i0 + m;
  const int v = visible_entries(q_pos[row], r, nc);
  const int full = v / block;
  const bool partial = (v % block) != 0;
  const int k1 = top_m - (partial ? 1 : 0);
  int* out = blk + ((size_t)b * nq + m) * top_m;
  if (k1 > 0) {
    select_row_reg_any<THREADS>(SB + ((size_t)b * nq + m) * ldB, full, k1, top_m, out, IdentityMap{}, sh);
  } else {
    for (int i = threadIdx.x; i < top_m; i += THREADS) out[i] = -1;
  }
  __syncthreads();
  if (partial && threadIdx.x == 0) out[full < k1 ? full : k1] = full;
}

// HISA stage 2: the k best candidates; candidate p is entry blocks[p / B] * B + p % B.
template <int THREADS>
__global__ void __launch_bounds__(THREADS, THREADS <= 256 ? 4 : 1)
select_cand_reg_kernel(const float* __restrict__ SC, const int* __restrict__ n_cand, const int* __restrict__ blk,
                       int* __restrict__ idx, int T_, int i0, int nq, int block, int top_m, int k) {
  __shared__ RegSelSmem<THREADS> sh;
  const int b = blockIdx.y, m = blockIdx.x;
  const size_t row = (size_t)b * T_ + i0 + m;
  const size_t slot = (size_t)b * nq + m;
  select_row_reg_any<THREADS>(SC + slot * ((size_t)top_m * block), n_cand[slot], k, k, idx + row * k,
                              BlockListMap{blk + slot * top_m, block}, sh);
}

}  // namespace hyb
