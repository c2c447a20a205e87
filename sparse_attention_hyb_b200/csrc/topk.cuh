// Top-k selection (HISA write-up, section 01: keep the k highest-scoring
// entries per query; ties go to the lower index).
//
// One CTA per query row.  The row's fp32 scores are mapped to order-preserving
// uint32 keys and copied into shared memory (when they fit), then an exact
// radix select finds the k-th largest key K* in four 8-bit passes (histogram
// with shared atomics, digit search with warp shuffles), and one ordered
// compaction pass writes every index with key > K* plus the lowest-index
// elements equal to K*, in ascending index order (warp ballot + popc prefix).
#pragma once
#include "common.cuh"

namespace hyb {

constexpr int kTopkThreads = 512;
constexpr int kTopkWarps = kTopkThreads / 32;

// Order-preserving map of fp32 to uint32 (both zeros map to the key of +0).
__device__ __forceinline__ uint32_t score_key(float f) {
  uint32_t u = __float_as_uint(f == 0.f ? 0.f : f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

struct TopkShared {
  uint32_t hist[256];
  uint32_t warp_gt[kTopkWarps];
  uint32_t warp_eq[kTopkWarps];
  uint32_t prefix;
  uint32_t remaining;
};

// Exact k-th largest key among keys[0..n) (n > k >= 1).  Returns K* and, in
// *need, how many elements equal to K* belong to the top k.
__device__ uint32_t radix_kth(const uint32_t* keys, int n, int k, TopkShared& sh, uint32_t* need) {
  const int tid = threadIdx.x;
  if (tid == 0) { sh.prefix = 0; sh.remaining = (uint32_t)k; }
  uint32_t mask = 0;
#pragma unroll 1
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int i = tid; i < 256; i += blockDim.x) sh.hist[i] = 0;
    __syncthreads();
    const uint32_t prefix = sh.prefix;
    for (int i = tid; i < n; i += blockDim.x) {
      const uint32_t key = keys[i];
      if ((key & mask) == prefix) atomicAdd(&sh.hist[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (tid < 32) {
      const int lane = tid;
      uint32_t h[8], tot = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) { h[e] = sh.hist[lane * 8 + e]; tot += h[e]; }
      // above = sum of totals of higher lanes (bins above this lane's range)
      uint32_t incl = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_down_sync(0xffffffffu, incl, o);
        if (lane + o < 32) incl += v;
      }
      uint32_t above = incl - tot;
      const uint32_t rem = sh.remaining;
      if (above < rem && rem <= incl) {
#pragma unroll
        for (int e = 7; e >= 0; --e) {
          if (above + h[e] >= rem) {
            sh.prefix = prefix | ((uint32_t)(lane * 8 + e) << shift);
            sh.remaining = rem - above;
            break;
          }
          above += h[e];
        }
      }
    }
    mask |= 255u << shift;
    __syncthreads();
  }
  *need = sh.remaining;
  return sh.prefix;
}

// Writes, in ascending position order, the positions p < n with key > kth and the
// first `need` positions with key == kth, as out[slot] = map(p).
template <typename Map>
__device__ void ordered_compact(const uint32_t* keys, int n, uint32_t kth, uint32_t need,
                                TopkShared& sh, int* out, Map map) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t base = 0, eq_seen = 0;
  for (int c0 = 0; c0 < n; c0 += blockDim.x) {
    const int i = c0 + tid;
    const uint32_t key = i < n ? keys[i] : 0u;
    const bool gt = i < n && key > kth;
    const bool eq = i < n && key == kth;
    const uint32_t bgt = __ballot_sync(0xffffffffu, gt), beq = __ballot_sync(0xffffffffu, eq);
    const uint32_t lt_mask = (1u << lane) - 1u;
    if (lane == 0) { sh.warp_gt[warp] = __popc(bgt); sh.warp_eq[warp] = __popc(beq); }
    __syncthreads();
    uint32_t gt_before = __popc(bgt & lt_mask), eq_before = __popc(beq & lt_mask);
    uint32_t gt_total = 0, eq_total = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
      const uint32_t g = sh.warp_gt[w], e = sh.warp_eq[w];
      if (w < warp) { gt_before += g; eq_before += e; }
      gt_total += g;
      eq_total += e;
    }
    const uint32_t eq_left = need > eq_seen ? need - eq_seen : 0u;
    if (gt || (eq && eq_before < eq_left)) {
      const uint32_t slot = base + gt_before + (eq_before < eq_left ? eq_before : eq_left);
      out[slot] = map(i);
    }
    base += gt_total + (eq_total < eq_left ? eq_total : eq_left);
    eq_seen += eq_total;
    __syncthreads();
  }
}

// Selects the k best of scores[0..n) into out[0..k) (k_out slots; -1 padding).
// keys_smem (if non-null) holds room for n keys; otherwise keys are read from
// scratch_keys (global memory, same length).
template <typename Map>
__device__ void select_row(const float* __restrict__ scores, int n, int k, int k_out,
                           uint32_t* keys, TopkShared& sh, int* out, Map map) {
  const int tid = threadIdx.x;
  if (n <= k) {
    for (int i = tid; i < k_out; i += blockDim.x) out[i] = i < n ? map(i) : -1;
    return;
  }
  for (int i = tid; i < n; i += blockDim.x) keys[i] = score_key(scores[i]);
  for (int i = k + tid; i < k_out; i += blockDim.x) out[i] = -1;
  __syncthreads();
  uint32_t need;
  const uint32_t kth = radix_kth(keys, n, k, sh, &need);
  ordered_compact(keys, n, kth, need, sh, out, map);
}

struct IdentityMap {
  __device__ __forceinline__ int operator()(int p) const { return p; }
};

// Candidate position -> entry id for HISA stage 2: candidates are laid out
// block by block in ascending block order, B per block.
struct BlockListMap {
  const int* blocks;
  int B;
  __device__ __forceinline__ int operator()(int p) const { return blocks[p / B] * B + p % B; }
};

}  // namespace hyb
