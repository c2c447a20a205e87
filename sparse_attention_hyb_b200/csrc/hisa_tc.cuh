// HISA stage 2 grouped by block (HISA write-up, section 02: the second stage
// scores only the entries of each query's selected blocks).  Within a query
// chunk every block is chosen by many queries, so instead of one gathered dot
// product per (query, entry) the work is regrouped per block:
//   hisa_count_kernel,     invert the per-query block lists (select_blocks
//   hisa_offsets_kernel,   output) into per-block lists of (query, slot) pairs:
//   hisa_scatter_kernel    per-block counts and each query's candidate count,
//                          list offsets and work items of up to kHgQ queries of
//                          one block, then the scatter (all grid-wide except the
//                          per-batch scan);
//   hisa_block_mma_kernel  one CTA per work item: the block's 128 entry keys
//                          (one 2-D TMA tile, 128-byte swizzle) times the
//                          item's query rows (16-byte cp.async gather) on the
//                          5th-generation tensor cores, M=128 entries x N=32
//                          queries x K=dI, fp32 accumulators in 32 TMEM columns;
//                          the scores land in the same candidate layout as the
//                          per-query scorer (row of the query, slot * block + e).
// Each block's keys are then read once per work item instead of once per query.
#pragma once
#include "common.cuh"
#include "sm100.cuh"

#include <type_traits>

namespace hyb {

constexpr int kHgQ = 32;             // queries per work item (MMA N)
constexpr int kHgBlock = 128;        // entries per block (MMA M)
constexpr int kHgMaxBlocks = 4096;   // blocks per batch handled by the grouping kernels
constexpr int kHgThreads = 1024;

// Work item: block g, list range [start, start + n) of the block's (query, slot) pairs.
struct HgWork {
  int g, start, n, pad;
};

// Upper bound of the work items of one batch: sum over blocks of ceil(count / kHgQ).
inline int hisa_work_cap(int nq, int top_m, int nb) { return (nq * top_m + kHgQ - 1) / kHgQ + nb; }

// Exclusive scan over the CTA (kHgThreads threads) of one value per thread.
__device__ __forceinline__ int hg_block_scan(int v, int* warp_tot, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += u;
  }
  __syncthreads();
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int t = warp_tot[lane];
    int ti = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, ti, o);
      if (lane >= o) ti += u;
    }
    warp_tot[lane] = ti - t;          // exclusive prefix of the warp totals
    if (lane == 31) warp_tot[32] = ti;
  }
  __syncthreads();
  total = warp_tot[32];
  return warp_tot[warp] + incl - v;
}

// Clears the per-block counters (before the first chunk; later chunks find them
// cleared by hisa_offsets_kernel).
__global__ void hisa_zero_kernel(int* __restrict__ cnt, int n) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) cnt[i] = 0;
}

// Warp per query row: counts the row's blocks into cnt[b][g] and writes the
// number of candidates of the row (the valid prefix of its candidate row).
__global__ void __launch_bounds__(256)
hisa_count_kernel(const int* __restrict__ q_pos, const int* __restrict__ blk, int* __restrict__ n_cand,
                  int* __restrict__ cnt, int T_, int i0, int nq, int r, int nc, int block, int top_m, int nbs) {
  const int b = blockIdx.y, lane = threadIdx.x & 31;
  const int m = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (m >= nq) return;
  const int* bl = blk + ((size_t)b * nq + m) * top_m;
  const int v = visible_entries(q_pos[(size_t)b * T_ + i0 + m], r, nc);
  int n2 = 0;
  for (int s = lane; s < top_m; s += 32) {
    const int g = bl[s];
    if (g >= 0 && g < nbs) {
      atomicAdd(&cnt[(size_t)b * nbs + g], 1);
      const int rem = v - g * block;
      n2 += rem < block ? rem : block;
    }
  }
  n2 = warp_sum(n2);
  if (lane == 0) n_cand[(size_t)b * nq + m] = n2;
}

// One CTA per batch: list offsets (fill[b][g], the scatter cursor of block g) and the
// work items (up to kHgQ queries of one block each); clears the counts.
__global__ void __launch_bounds__(kHgThreads)
hisa_offsets_kernel(int* __restrict__ cnt, int* __restrict__ fill, HgWork* __restrict__ work,
                    int* __restrict__ n_work, int nbs, int work_cap) {
  __shared__ int warp_tot[33];
  const int b = blockIdx.x, tid = threadIdx.x;
  constexpr int kPer = kHgMaxBlocks / kHgThreads;
  const int g0 = tid * kPer;
  int c[kPer];
  int c_sum = 0, t_sum = 0;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int g = g0 + i;
    c[i] = g < nbs ? cnt[(size_t)b * nbs + g] : 0;
    c_sum += c[i];
    t_sum += (c[i] + kHgQ - 1) / kHgQ;
  }
  int c_tot, t_tot;
  int c_off = hg_block_scan(c_sum, warp_tot, c_tot);
  int t_off = hg_block_scan(t_sum, warp_tot, t_tot);
  HgWork* wb = work + (size_t)b * work_cap;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int g = g0 + i;
    if (g >= nbs) break;
    fill[(size_t)b * nbs + g] = c_off;
    cnt[(size_t)b * nbs + g] = 0;
    for (int t = 0; t * kHgQ < c[i]; ++t) {
      const int n = c[i] - t * kHgQ;
      wb[t_off + t] = HgWork{g, c_off + t * kHgQ, n < kHgQ ? n : kHgQ, 0};
    }
    c_off += c[i];
    t_off += (c[i] + kHgQ - 1) / kHgQ;
  }
  if (tid == 0) n_work[b] = t_tot;
}

// (query, slot) pairs into their block's list; p = m * top_m + s.
__global__ void __launch_bounds__(256)
hisa_scatter_kernel(const int* __restrict__ blk, int* __restrict__ fill, int* __restrict__ list, int nq, int top_m,
                    int nbs) {
  const int b = blockIdx.y;
  const int p = blockIdx.x * 256 + threadIdx.x;
  if (p >= nq * top_m) return;
  const size_t base = (size_t)b * nq * top_m;
  const int g = blk[base + p];
  if (g >= 0 && g < nbs) list[base + atomicAdd(&fill[(size_t)b * nbs + g], 1)] = p;
}

template <int KB>  // dI = 64 * KB
struct HgSmem {
  static constexpr int kK = KB * kHgBlock * 128;   // entry keys, 64-column sub-tiles of 128 rows
  static constexpr int kQ = KB * kHgQ * 128;       // query rows, 64-column sub-tiles of 32 rows
  static constexpr int kTotal = kK + kQ + 1024;
};

template <typename T, int KB>
__global__ void __launch_bounds__(128)
hisa_block_mma_kernel(const __grid_constant__ CUtensorMap map_ic, const T* __restrict__ qi,
                      const int* __restrict__ list, const HgWork* __restrict__ work, const int* __restrict__ n_work,
                      float* __restrict__ SC, int T_, int i0, int nq, int nc_cap, int top_m, int work_cap) {
  using namespace sm100;
  using L = HgSmem<KB>;
  constexpr int dI = 64 * KB;
  const int b = blockIdx.y, w = blockIdx.x;
  if (w >= n_work[b]) return;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = smem;
  uint8_t* sQ = smem + L::kK;
  __shared__ uint64_t bar_k, bar_mma;
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;
  __shared__ int qm[kHgQ], qs[kHgQ];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const HgWork it = work[(size_t)b * work_cap + w];
  if (tid == 0) {
    abort_flag = 0;
    mbar_init(&bar_k, 1);
    mbar_init(&bar_mma, 1);
    fence_mbar_init();
  }
  if (tid < kHgQ) {
    const int p = tid < it.n ? list[(size_t)b * nq * top_m + it.start + tid] : 0;
    qm[tid] = p / top_m;
    qs[tid] = p % top_m;
  }
  if (warp == 0) tmem_alloc(&tmem_base, 32);
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = tmem_base;
  if (tid == 0) {
    prefetch_tmap(&map_ic);
    mbar_expect_tx(&bar_k, L::kK);
    for (int c = 0; c < KB; ++c)
      tma_load_2d(sK + c * (kHgBlock * 128), &map_ic, &bar_k, c * 64, b * nc_cap + it.g * kHgBlock);
  }
  // query rows: 16-byte chunks written in the 128-byte swizzle; rows past n are zero
  const T* qbase = qi + ((size_t)b * T_ + i0) * dI;
  for (int u = tid; u < kHgQ * 8 * KB; u += 128) {
    const int j = u / (8 * KB), c = (u / 8) % KB, ch = u % 8;
    const bool real = j < it.n;
    const T* src = qbase + (size_t)(real ? qm[j] : 0) * dI + c * 64 + ch * 8;
    cp_async16_zfill(smem_u32(sQ + c * (kHgQ * 128) + j * 128 + ((ch ^ (j & 7)) << 4)), src, real ? 16u : 0u);
  }
  cp_async_commit();
  cp_async_wait<0>();
  fence_async_shared();
  __syncthreads();
  if (tid == 0) {
    if (mbar_wait(&bar_k, 0, &abort_flag)) {
      fence_after_sync();
      constexpr uint32_t idesc = idesc_bf16_f32(kHgBlock, kHgQ);
#pragma unroll
      for (int c = 0; c < KB; ++c)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_f16_ss(tmem, desc_kmajor_sw128(smem_u32(sK + c * (kHgBlock * 128) + kk * 32)),
                     desc_kmajor_sw128(smem_u32(sQ + c * (kHgQ * 128) + kk * 32)), idesc, (c | kk) != 0);
    }
    mma_commit(&bar_mma);   // arrives once the issued MMAs (if any) are complete
  }
  const bool ok = mbar_wait(&bar_mma, 0, &abort_flag);
  fence_after_sync();
  if (ok && !abort_flag) {
    uint32_t v[32];
    tmem_ld32(tmem + (static_cast<uint32_t>(warp * 32) << 16), v);
    tmem_wait_ld();
    const int e = warp * 32 + lane;   // entry of the block
    const size_t row_len = (size_t)top_m * kHgBlock;
#pragma unroll 4
    for (int j = 0; j < kHgQ; ++j)
      if (j < it.n) SC[((size_t)b * nq + qm[j]) * row_len + (size_t)qs[j] * kHgBlock + e] = __uint_as_float(v[j]);
  }
  fence_before_sync();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 32);
}

// The grouped stage 2 needs bf16 keys with 128-entry blocks, dI of 64 or 128,
// 16-byte aligned query and key rows, and at most kHgMaxBlocks blocks
// (counting the partial one).
template <typename T>
inline bool hisa_grouped_supported(int dI, int block, int nb, const void* qi, const void* ic) {
  auto al = [](const void* p) { return reinterpret_cast<uintptr_t>(p) % 16 == 0; };
  return std::is_same<T, bf16>::value && block == kHgBlock && (dI == 64 || dI == 128) && nb + 1 <= kHgMaxBlocks &&
         al(qi) && al(ic);
}

inline cudaError_t launch_hisa_block_mma(const void* qi, const void* ic, const int* list, const HgWork* work,
                                         const int* n_work, float* SC, int batch, int T_, int i0, int nq, int dI,
                                         int nc_cap, int top_m, int work_cap, cudaStream_t stream) {
  CUtensorMap m;
  if (!make_map_bf16_2d(&m, ic, (uint64_t)batch * nc_cap, dI, (uint64_t)dI * 2, kHgBlock, 64))
    return cudaErrorInvalidValue;
  const dim3 grid(work_cap, batch);
  if (dI == 128) {
    hisa_block_mma_kernel<bf16, 2><<<grid, 128, HgSmem<2>::kTotal, stream>>>(m, (const bf16*)qi, list, work, n_work,
                                                                             SC, T_, i0, nq, nc_cap, top_m, work_cap);
  } else {
    hisa_block_mma_kernel<bf16, 1><<<grid, 128, HgSmem<1>::kTotal, stream>>>(m, (const bf16*)qi, list, work, n_work,
                                                                             SC, T_, i0, nq, nc_cap, top_m, work_cap);
  }
  count_launch();
  return cudaGetLastError();
}

}  // namespace hyb
