// Indexer scores on the 5th-generation tensor cores (bf16 operands, fp32
// accumulation in tensor memory): S[row, j] = q_I[row] . keys[j] for a chunk of
// query rows (HISA write-up, section 01: every query scores every prefix entry;
// the same kernel scores HISA block representatives in stage 1).
//
// One CTA owns 128 query rows (the M of one tcgen05.mma) and walks a strided
// subset of the 256-entry column tiles its rows can see:
//   warp 0      TMA producer: the 128 x dI query tile once, then key tiles
//               (256 x dI, 128-byte swizzle) into a 2-stage ring;
//   warp 1      allocates 512 TMEM columns; one thread issues the MMAs
//               (M=128, N=256, K=16 steps) into one of two 256-column
//               accumulators and commits them to the ring / epilogue barriers;
//   warps 2..5  epilogue: tcgen05.ld 32 columns at a time from their lane
//               quadrant, stage each 32 x 32 fp32 block in shared memory
//               (128-byte swizzle, four buffers per warp) and write it with a
//               TMA tensor store, so the scores leave as whole lines.
// Column tiles no row of the CTA can see are never loaded (causal skipping).
#pragma once
#include "common.cuh"
#include "sm100.cuh"

namespace hyb {

constexpr int kTcBM = 128;
constexpr int kTcBN = 256;
constexpr int kTcStages = 2;
constexpr int kTcThreads = 192;

template <int KB>  // dI = 64 * KB
struct TcScoreSmem {
  static constexpr int kA = KB * kTcBM * 128;          // bytes of the query tile
  static constexpr int kB = KB * kTcBN * 128;          // bytes of one key tile
  static constexpr int kStg = 4;                       // staging buffers per epilogue warp
  static constexpr int kC = 4 * kStg * 32 * 128;       // epilogue staging: 4 warps x kStg buffers x 32 rows x 128 B
  static constexpr int kTotal = kA + kTcStages * kB + kC + 1024;  // + alignment slack
};

template <int KB>
__global__ void __launch_bounds__(kTcThreads, 1)
scores_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                 const __grid_constant__ CUtensorMap map_s, const int* __restrict__ q_pos, int T_, int i0, int nq, int keys_cap,
                 int r, int nc, int div, int ldS, int nsplit) {
  using namespace sm100;
  using L = TcScoreSmem<KB>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + L::kA;
  uint8_t* sC = sB + kTcStages * L::kB;
  __shared__ uint64_t bar_a, bar_full[kTcStages], bar_empty[kTcStages], bar_tfull[2], bar_tempty[2], bar_done;
  __shared__ uint32_t tmem_base;
  __shared__ int tile_cols;
  __shared__ int abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // query tiles last first: in causal order they see the most keys
  const int b = blockIdx.z, m0 = (int)(gridDim.x - 1 - blockIdx.x) * kTcBM, split = blockIdx.y;

  if (tid == 0) {
    tile_cols = 0;
    abort_flag = 0;
    mbar_init(&bar_a, 1);
    for (int s = 0; s < kTcStages; ++s) { mbar_init(&bar_full[s], 1); mbar_init(&bar_empty[s], 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(&bar_tfull[a], 1); mbar_init(&bar_tempty[a], 4); }
    mbar_init(&bar_done, 1);
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(&tmem_base, 512);
  __syncthreads();
  if (tid < kTcBM && m0 + tid < nq) {
    const int t = q_pos[(size_t)b * T_ + i0 + m0 + tid];
    atomicMax(&tile_cols, visible_entries(t, r, nc) / div);
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const int cols = tile_cols;
  const int n_tiles = (cols + kTcBN - 1) / kTcBN;
  const int my_tiles = split < n_tiles ? (n_tiles - split + nsplit - 1) / nsplit : 0;
  const uint32_t tmem = tmem_base;
  constexpr uint32_t kIdesc = idesc_bf16_f32(kTcBM, kTcBN);

  if (my_tiles > 0) {
    if (warp == 0 && lane == 0) {
      // ---------------- producer
      prefetch_tmap(&map_q);
      prefetch_tmap(&map_k);
      mbar_expect_tx(&bar_a, L::kA);
      for (int kb = 0; kb < KB; ++kb)
        tma_load_2d(sA + kb * kTcBM * 128, &map_q, &bar_a, kb * 64, b * T_ + i0 + m0);
      int issued = 0;
      for (int it = 0; it < my_tiles; ++it) {
        const int s = it % kTcStages;
        const uint32_t ph = (it / kTcStages) & 1;
        if (!mbar_wait(&bar_empty[s], ph ^ 1, &abort_flag)) break;
        const int n = split + it * nsplit;
        mbar_expect_tx(&bar_full[s], L::kB);
        for (int kb = 0; kb < KB; ++kb)
          tma_load_2d(sB + s * L::kB + kb * kTcBN * 128, &map_k, &bar_full[s], kb * 64, b * keys_cap + n * kTcBN);
        ++issued;
      }
      if (abort_flag) {
        // drain: every issued load must land before the CTA may exit
        unsigned long long t0 = globaltimer();
        for (int it = 0; it < issued; ++it) {
          const int s = it % kTcStages;
          const uint32_t ph = (it / kTcStages) & 1;
          while (!mbar_try_wait(&bar_full[s], ph) && globaltimer() - t0 < kWaitNs) {}
        }
        while (!mbar_try_wait(&bar_a, 0) && globaltimer() - t0 < kWaitNs) {}
      }
    } else if (warp == 1 && lane == 0) {
      // ---------------- MMA issuer
      if (mbar_wait(&bar_a, 0, &abort_flag)) {
        for (int it = 0; it < my_tiles; ++it) {
          const int s = it % kTcStages;
          const uint32_t ph = (it / kTcStages) & 1;
          const int acc = it & 1;
          const uint32_t aph = (it >> 1) & 1;
          if (!mbar_wait(&bar_full[s], ph, &abort_flag)) break;
          if (!mbar_wait(&bar_tempty[acc], aph ^ 1, &abort_flag)) break;
          fence_after_sync();
          const uint32_t d = tmem + acc * kTcBN;
#pragma unroll
          for (int kb = 0; kb < KB; ++kb) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t ad = desc_kmajor_sw128(smem_u32(sA + kb * kTcBM * 128 + kk * 32));
              const uint64_t bd = desc_kmajor_sw128(smem_u32(sB + s * L::kB + kb * kTcBN * 128 + kk * 32));
              mma_f16_ss(d, ad, bd, kIdesc, (kb | kk) != 0);
            }
          }
          mma_commit(&bar_empty[s]);
          mma_commit(&bar_tfull[acc]);
        }
      }
      // all issued MMAs complete before TMEM is released
      mma_commit(&bar_done);
      unsigned long long t0 = globaltimer();
      while (!mbar_try_wait(&bar_done, 0) && globaltimer() - t0 < kWaitNs) {}
    } else if (warp >= 2) {
      // ---------------- epilogue
      const int quad = warp & 3;
      uint8_t* stg = sC + quad * (L::kStg * 32 * 128);
      uint32_t nst = 0;   // blocks this warp has stored
      for (int it = 0; it < my_tiles; ++it) {
        const int acc = it & 1;
        const uint32_t aph = (it >> 1) & 1;
        if (!mbar_wait(&bar_tfull[acc], aph, &abort_flag)) break;
        fence_after_sync();
        const int col0 = (split + it * nsplit) * kTcBN;
#pragma unroll 1
        for (int c = 0; c < kTcBN / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(tmem + (static_cast<uint32_t>(quad * 32) << 16) + acc * kTcBN + c * 32, v);
          tmem_wait_ld();
          const int cb = col0 + c * 32;
          if (cb >= cols || m0 + quad * 32 >= nq) continue;   // columns no row can see; rows past the chunk
          uint8_t* buf = stg + (nst % L::kStg) * (32 * 128);
          if (nst >= L::kStg && lane == 0) bulk_wait_read<L::kStg - 1>();   // the store kStg blocks back has read this buffer
          __syncwarp();
#pragma unroll
          for (int e = 0; e < 8; ++e)
            *reinterpret_cast<uint4*>(buf + lane * 128 + ((e ^ (lane & 7)) << 4)) =
                make_uint4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
          fence_async_shared();
          __syncwarp();
          if (lane == 0) {
            tma_store_3d(&map_s, smem_u32(buf), cb, m0 + quad * 32, b);   // rows past nq are clipped
            bulk_commit();
          }
          ++nst;
        }
        fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar_tempty[acc]);
      }
      if (lane == 0) bulk_wait_all();
    }
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// Host: scores for query rows [i0, i0 + nq) of every batch into S (row stride
// ldS).  keys: [batch, keys_cap, dI] bf16; qi: [batch, T, dI] bf16.  Returns
// false when the shapes are not handled by this kernel (the caller then uses
// the CUDA-core scorer).
inline bool tc_scores_supported(int dI, const void* qi, const void* keys) {
  return (dI == 64 || dI == 128) && (reinterpret_cast<uintptr_t>(qi) % 16 == 0) &&
         (reinterpret_cast<uintptr_t>(keys) % 16 == 0);
}

inline cudaError_t launch_scores_tc(const void* qi, const int* q_pos, const void* keys, float* S, int batch, int T_,
                                    int i0, int nq, int dI, int keys_cap, int r, int nc, int div, int ldS,
                                    int max_cols, cudaStream_t stream) {
  CUtensorMap mq, mk, ms;
  if (!make_map_bf16_2d(&mq, qi, (uint64_t)batch * T_, dI, (uint64_t)dI * 2, kTcBM, 64)) return cudaErrorInvalidValue;
  if (!make_map_bf16_2d(&mk, keys, (uint64_t)batch * keys_cap, dI, (uint64_t)dI * 2, kTcBN, 64))
    return cudaErrorInvalidValue;
  if (!make_map_f32_3d(&ms, S, (uint64_t)ldS, (uint64_t)ldS, (uint64_t)nq, (uint64_t)batch, 32)) return cudaErrorInvalidValue;
  const int m_tiles = (nq + kTcBM - 1) / kTcBM;
  const int n_tiles = (max_cols + kTcBN - 1) / kTcBN;
  int nsplit = (2 * 148 + m_tiles * batch - 1) / (m_tiles * batch);
  if (nsplit > n_tiles) nsplit = n_tiles;
  if (nsplit < 1) nsplit = 1;
  dim3 grid(m_tiles, nsplit, batch);
  cudaError_t e;
  if (dI == 128) {
    const int smem = TcScoreSmem<2>::kTotal;
    if ((e = cudaFuncSetAttribute(scores_tc_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) != cudaSuccess)
      return e;
    scores_tc_kernel<2><<<grid, kTcThreads, smem, stream>>>(mq, mk, ms, q_pos, T_, i0, nq, keys_cap, r, nc, div,
                                                             ldS, nsplit);
  } else {
    const int smem = TcScoreSmem<1>::kTotal;
    if ((e = cudaFuncSetAttribute(scores_tc_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) != cudaSuccess)
      return e;
    scores_tc_kernel<1><<<grid, kTcThreads, smem, stream>>>(mq, mk, ms, q_pos, T_, i0, nq, keys_cap, r, nc, div,
                                                             ldS, nsplit);
  }
  count_launch();
  return cudaGetLastError();
}

}  // namespace hyb
