// S2 — indexer scores and top-k selection, flat and HISA two-stage (HISA
// write-up, sections 01 and 02).  CUDA-core (FFMA) implementations: these are
// the path for fp32 inputs and the baseline the tensor-core scorer replaces
// for bf16.
#pragma once
#include <type_traits>
#include "common.cuh"
#include "topk.cuh"

namespace hyb {

// Score tile geometry of the FFMA scorer.
constexpr int kSB_M = 64, kSB_N = 64, kSB_K = 32;

// Number of score columns row (b, i) needs: visible entries (div = 1) or
// visible full blocks (div = block).
__device__ __forceinline__ int score_cols(int t, int r, int nc, int div) {
  return visible_entries(t, r, nc) / div;
}

// Same scores for chunks of one or two query rows per batch (decode): streaming
// the keys once is the whole cost, so each warp takes 32 consecutive keys (fully
// unrolled, so their loads are in flight together), every lane holds dI/32
// channels of the query row(s), and one transposed warp reduction leaves key
// j0+l's score in lane l (a coalesced 128-byte store per warp and row).
constexpr int kGvKeys = 256;   // keys per CTA: 8 warps x 32

template <int N>
__device__ __forceinline__ void gv_xsum_step(float* v, int lane, int mask) {
  const bool hi = (lane & mask) != 0;
#pragma unroll
  for (int i = 0; i < N / 2; ++i) {
    const float send = hi ? v[i] : v[i + N / 2];
    const float keep = hi ? v[i + N / 2] : v[i];
    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, mask);
  }
}

template <typename T, int DPL>
__device__ __forceinline__ void gv_load(const T* p, float (&x)[DPL]) {
  if constexpr (std::is_same<T, float>::value) {
    static_assert(DPL % 2 == 0, "");
#pragma unroll
    for (int e = 0; e < DPL; e += 2) {
      const float2 v = *reinterpret_cast<const float2*>(p + e);
      x[e] = v.x; x[e + 1] = v.y;
    }
  } else {
#pragma unroll
    for (int e = 0; e < DPL; e += 2) {
      const __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(p + e);
      x[e] = __low2float(v); x[e + 1] = __high2float(v);
    }
  }
}

template <typename T, int DPL, int NQ>   // DPL = dI / 32 channels per lane; NQ query rows (1 or 2)
__global__ void __launch_bounds__(256)
scores_gemv_kernel(const T* __restrict__ qi, const int* __restrict__ q_pos, const T* __restrict__ keys,
                   float* __restrict__ S, int T_, int i0, int keys_cap, int r, int nc, int div, int ldS) {
  constexpr int dI = DPL * 32;
  const int b = blockIdx.y, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float q[NQ][DPL];
  int cols[NQ];
  int maxc = 0;
#pragma unroll
  for (int m = 0; m < NQ; ++m) {
    const size_t row = (size_t)b * T_ + i0 + m;
    cols[m] = score_cols(q_pos[row], r, nc, div);
    maxc = cols[m] > maxc ? cols[m] : maxc;
    gv_load<T, DPL>(qi + row * dI + lane * DPL, q[m]);
  }
  const int j0 = blockIdx.x * kGvKeys + warp * 32;
  if (j0 >= maxc) return;
  const T* kb = keys + (size_t)b * keys_cap * dI + lane * DPL;
  float part[NQ][32];
#pragma unroll
  for (int u = 0; u < 32; ++u) {
    float kv[DPL];
    if (j0 + u < maxc) {
      gv_load<T, DPL>(kb + (size_t)(j0 + u) * dI, kv);
    } else {
#pragma unroll
      for (int e = 0; e < DPL; ++e) kv[e] = 0.f;
    }
#pragma unroll
    for (int m = 0; m < NQ; ++m) {
      float acc = 0.f;
#pragma unroll
      for (int e = 0; e < DPL; ++e) acc = fmaf(q[m][e], kv[e], acc);
      part[m][u] = acc;
    }
  }
#pragma unroll
  for (int m = 0; m < NQ; ++m) {
    gv_xsum_step<32>(part[m], lane, 16); gv_xsum_step<16>(part[m], lane, 8); gv_xsum_step<8>(part[m], lane, 4);
    gv_xsum_step<4>(part[m], lane, 2); gv_xsum_step<2>(part[m], lane, 1);
    const int j = j0 + lane;
    if (j < cols[m]) S[((size_t)b * NQ + m) * ldS + j] = part[m][0];
  }
}

// bf16 variant of the same scores with 16-byte loads: LPK = dI / 8 lanes hold one
// key row, so each load instruction of a warp covers 32 / LPK keys and a warp's 32
// keys take LPK loads per lane, all in flight together.  The transposed reduction
// over the LPK lanes of a key leaves key j0 + (l % LPK) * (32 / LPK) + l / LPK in
// lane l (the warp's 32 scores in one 128-byte segment).
// Eight bf16 (a 16-byte vector, lowest address first) to fp32: a bf16 is the upper
// half of the fp32 with the same value.
__device__ __forceinline__ void bf16x8_to_f32(const uint4 v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    f[2 * e] = __uint_as_float(w[e] << 16);
    f[2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
  }
}

template <int LPK, int NQ>
__global__ void __launch_bounds__(256)
scores_gemv16_kernel(const bf16* __restrict__ qi, const int* __restrict__ q_pos, const bf16* __restrict__ keys,
                     float* __restrict__ S, int T_, int i0, int keys_cap, int r, int nc, int div, int ldS) {
  constexpr int dI = LPK * 8, KPI = 32 / LPK;
  const int b = blockIdx.y, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = lane % LPK, kofs = lane / LPK;
  float q[NQ][8];
  int cols[NQ];
  int maxc = 0;
#pragma unroll
  for (int m = 0; m < NQ; ++m) {
    const size_t row = (size_t)b * T_ + i0 + m;
    cols[m] = score_cols(q_pos[row], r, nc, div);
    maxc = cols[m] > maxc ? cols[m] : maxc;
    bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(qi + row * dI + sub * 8)), q[m]);
  }
  const int j0 = blockIdx.x * kGvKeys + warp * 32;
  if (j0 >= maxc) return;
  const bf16* kb = keys + (size_t)b * keys_cap * dI + sub * 8;
  uint4 raw[LPK];
#pragma unroll
  for (int i = 0; i < LPK; ++i) {
    const int j = j0 + i * KPI + kofs;
    raw[i] = j < maxc ? __ldg(reinterpret_cast<const uint4*>(kb + (size_t)j * dI)) : make_uint4(0, 0, 0, 0);
  }
  float part[NQ][LPK];
#pragma unroll
  for (int i = 0; i < LPK; ++i) {
    float kv[8];
    bf16x8_to_f32(raw[i], kv);
#pragma unroll
    for (int m = 0; m < NQ; ++m) {
      float acc = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) acc = fmaf(q[m][e], kv[e], acc);
      part[m][i] = acc;
    }
  }
#pragma unroll
  for (int m = 0; m < NQ; ++m) {
    if constexpr (LPK == 16) gv_xsum_step<16>(part[m], lane, 8);
    gv_xsum_step<8>(part[m], lane, 4);
    gv_xsum_step<4>(part[m], lane, 2);
    gv_xsum_step<2>(part[m], lane, 1);
    const int j = j0 + sub * KPI + kofs;
    if (j < cols[m]) S[((size_t)b * NQ + m) * ldS + j] = part[m][0];
  }
}

// S[b, i - i0, j] = qi[b, i] . keys[b, j] for j < score_cols(row), rows i in
// [i0, i0 + nq).  keys: [batch, keys_cap, dI].  Output row stride ldS.
// Tiles whose columns are all invisible to every row of the tile are skipped.
template <typename T>
__global__ void __launch_bounds__(256)
scores_ffma_kernel(const T* __restrict__ qi, const int* __restrict__ q_pos,
                   const T* __restrict__ keys, float* __restrict__ S, int T_, int i0, int nq,
                   int dI, int keys_cap, int r, int nc, int div, int ldS) {
  __shared__ float As[kSB_K][kSB_M + 4];
  __shared__ float Bs[kSB_K][kSB_N + 4];
  __shared__ int tile_cols;
  const int b = blockIdx.z;
  const int m0 = blockIdx.y * kSB_M, n0 = blockIdx.x * kSB_N;
  const int tid = threadIdx.x;
  if (tid == 0) tile_cols = 0;
  __syncthreads();
  if (tid < kSB_M && m0 + tid < nq) {
    const int t = q_pos[(size_t)b * T_ + i0 + m0 + tid];
    atomicMax(&tile_cols, score_cols(t, r, nc, div));
  }
  __syncthreads();
  if (n0 >= tile_cols) return;

  const int tx = tid & 15, ty = tid >> 4;  // 16 x 16 threads, 4 x 4 outputs each
  float acc[4][4] = {};
  const T* qb = qi + ((size_t)b * T_ + i0) * dI;
  const T* kb = keys + (size_t)b * keys_cap * dI;
  for (int k0 = 0; k0 < dI; k0 += kSB_K) {
    for (int e = tid; e < kSB_M * kSB_K; e += 256) {
      const int m = e / kSB_K, kk = e % kSB_K;
      As[kk][m] = (m0 + m < nq && k0 + kk < dI) ? to_f(qb[(size_t)(m0 + m) * dI + k0 + kk]) : 0.f;
      Bs[kk][m] = (n0 + m < tile_cols && k0 + kk < dI) ? to_f(kb[(size_t)(n0 + m) * dI + k0 + kk]) : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < kSB_K; ++kk) {
      float a[4], bv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) { a[u] = As[kk][ty * 4 + u]; bv[u] = Bs[kk][tx * 4 + u]; }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(a[u], bv[v], acc[u][v]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int m = m0 + ty * 4 + u;
    if (m >= nq) continue;
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int n = n0 + tx * 4 + v;
      if (n < tile_cols) S[((size_t)b * nq + m) * ldS + n] = acc[u][v];
    }
  }
}

// Flat selection: row (b, i) keeps the k best of its visible entries.
__global__ void __launch_bounds__(kTopkThreads)
select_flat_kernel(const float* __restrict__ S, const int* __restrict__ q_pos, int* __restrict__ idx,
                   int T_, int i0, int nq, int r, int nc, int k, int ldS, uint32_t* gkeys) {
  extern __shared__ uint32_t dyn_keys[];
  __shared__ TopkShared sh;
  const int b = blockIdx.y, m = blockIdx.x;
  const size_t row = (size_t)b * T_ + i0 + m;
  const int n = visible_entries(q_pos[row], r, nc);
  uint32_t* keys = gkeys ? gkeys + ((size_t)b * nq + m) * ldS : dyn_keys;
  select_row(S + ((size_t)b * nq + m) * ldS, n, k, k, keys, sh, idx + row * k, IdentityMap{});
}

// HISA stage 1 selection: the partial block (if any) is always kept; the best
// full blocks fill the other slots.  blk row: kept blocks ascending, then -1.
__global__ void __launch_bounds__(kTopkThreads)
select_blocks_kernel(const float* __restrict__ SB, const int* __restrict__ q_pos, int* __restrict__ blk,
                     int T_, int i0, int nq, int r, int nc, int block, int top_m, int ldB) {
  extern __shared__ uint32_t dyn_keys[];
  __shared__ TopkShared sh;
  const int b = blockIdx.y, m = blockIdx.x;
  const size_t row = (size_t)b * T_ + i0 + m;
  const int v = visible_entries(q_pos[row], r, nc);
  const int full = v / block;
  const bool partial = (v % block) != 0;
  const int k1 = top_m - (partial ? 1 : 0);
  int* out = blk + ((size_t)b * nq + m) * top_m;
  if (k1 > 0) {
    select_row(SB + ((size_t)b * nq + m) * ldB, full, k1, top_m, dyn_keys, sh, out, IdentityMap{});
  } else {
    for (int i = threadIdx.x; i < top_m; i += blockDim.x) out[i] = -1;
  }
  __syncthreads();
  if (partial && threadIdx.x == 0) out[full < k1 ? full : k1] = full;
}

// HISA stage 2 for a few queries (decode): one CTA per (query, kept block slot),
// one thread per entry of the block, so the whole candidate row is scored in one
// launch.  Candidate p of a query is entry blk[p / B] * B + p % B (the kept blocks
// in ascending order, the partial block last); slot 0 also writes the count.
template <typename T>
__global__ void __launch_bounds__(128)
hisa_slot_scores_kernel(const T* __restrict__ qi, const int* __restrict__ q_pos, const T* __restrict__ ic,
                        const int* __restrict__ blk, float* __restrict__ SC, int* __restrict__ n_cand, int T_, int i0,
                        int nq, int dI, int nc_cap, int r, int nc, int block, int top_m) {
  extern __shared__ float qrow[];
  const int slot = blockIdx.x, m = blockIdx.y, b = blockIdx.z;
  const size_t row = (size_t)b * T_ + i0 + m;
  const int v = visible_entries(q_pos[row], r, nc);
  const int* bl = blk + ((size_t)b * nq + m) * top_m;
  if (slot == 0 && threadIdx.x == 0) {
    int n2 = 0;
    for (int s = 0; s < top_m && bl[s] >= 0; ++s) {
      const int rem = v - bl[s] * block;
      n2 += rem < block ? rem : block;
    }
    n_cand[(size_t)b * nq + m] = n2;
  }
  const int g = bl[slot];
  if (g < 0) return;
  const int rem = v - g * block;
  const int cnt = rem < block ? rem : block;
  for (int c = threadIdx.x; c < dI; c += blockDim.x) qrow[c] = to_f(qi[row * dI + c]);
  __syncthreads();
  float* out = SC + ((size_t)b * nq + m) * ((size_t)top_m * block) + (size_t)slot * block;
  const T* icb = ic + ((size_t)b * nc_cap + (size_t)g * block) * dI;
  for (int e = threadIdx.x; e < cnt; e += blockDim.x) {
    const T* krow = icb + (size_t)e * dI;
    float acc = 0.f;
    for (int c = 0; c < dI; c += 4) {
      const float4 kv = load4(krow + c);
      acc = fmaf(qrow[c], kv.x, acc);
      acc = fmaf(qrow[c + 1], kv.y, acc);
      acc = fmaf(qrow[c + 2], kv.z, acc);
      acc = fmaf(qrow[c + 3], kv.w, acc);
    }
    out[e] = acc;
  }
}

// HISA stage 2 scores: candidate p of row (b, i) is entry blocks[p / B] * B + p % B;
// the valid candidates form a prefix of length n2 (blocks ascending, the
// partial block last).  One warp per candidate, lanes over channels.
template <typename T>
__global__ void __launch_bounds__(256)
hisa_cand_scores_kernel(const T* __restrict__ qi, const int* __restrict__ q_pos,
                        const T* __restrict__ ic, const int* __restrict__ blk, float* __restrict__ SC,
                        int* __restrict__ n_cand, int T_, int i0, int nq, int dI, int nc_cap, int r,
                        int nc, int block, int top_m) {
  extern __shared__ float qrow[];
  const int b = blockIdx.y, m = blockIdx.x;
  const size_t row = (size_t)b * T_ + i0 + m;
  const int v = visible_entries(q_pos[row], r, nc);
  const int* bl = blk + ((size_t)b * nq + m) * top_m;
  for (int c = threadIdx.x; c < dI; c += blockDim.x) qrow[c] = to_f(qi[row * dI + c]);
  __shared__ int s_n2;
  if (threadIdx.x == 0) {
    int n2 = 0;
    for (int s = 0; s < top_m && bl[s] >= 0; ++s) {
      const int rem = v - bl[s] * block;
      n2 += rem < block ? rem : block;
    }
    s_n2 = n2;
    n_cand[(size_t)b * nq + m] = n2;
  }
  __syncthreads();
  const int n2 = s_n2;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const T* icb = ic + (size_t)b * nc_cap * dI;
  float* out = SC + ((size_t)b * nq + m) * ((size_t)top_m * block);
  for (int p = warp; p < n2; p += blockDim.x >> 5) {
    const int j = bl[p / block] * block + p % block;
    const T* krow = icb + (size_t)j * dI;
    float acc = 0.f;
    for (int c = lane * 4; c < dI; c += 128) {
      const float4 kv = load4(krow + c);
      acc = fmaf(qrow[c], kv.x, acc);
      acc = fmaf(qrow[c + 1], kv.y, acc);
      acc = fmaf(qrow[c + 2], kv.z, acc);
      acc = fmaf(qrow[c + 3], kv.w, acc);
    }
    acc = warp_sum(acc);
    if (lane == 0) out[p] = acc;
  }
}

__global__ void __launch_bounds__(kTopkThreads)
select_cand_kernel(const float* __restrict__ SC, const int* __restrict__ n_cand,
                   const int* __restrict__ blk, int* __restrict__ idx, int T_, int i0, int nq,
                   int block, int top_m, int k) {
  extern __shared__ uint32_t dyn_keys[];
  __shared__ TopkShared sh;
  const int b = blockIdx.y, m = blockIdx.x;
  const size_t row = (size_t)b * T_ + i0 + m;
  const size_t slot = (size_t)b * nq + m;
  select_row(SC + slot * ((size_t)top_m * block), n_cand[slot], k, k, dyn_keys, sh, idx + row * k,
             BlockListMap{blk + slot * top_m, block});
}

}  // namespace hyb
