// S3 + S4 — shared-KV (MQA) attention over compressed entries plus the
// sliding window, one joint softmax (HCA article, section "怎么压"; trdm.cn 2.1).
//
// CUDA-core (FFMA) implementation: the path for fp32 inputs and the baseline
// the tensor-core kernels replace for bf16.  One CTA per query (all heads);
// keys are gathered 32 at a time into shared memory and consumed with a
// flash-style online softmax.  With nsplit > 1 each CTA handles a slice of the
// query's key list and writes a partial (o, lse) that attn_merge combines.
#pragma once
#include "common.cuh"

namespace hyb {

constexpr int kAttnThreads = 256;
constexpr int kAttnTile = 32;

struct AttnArgs {
  const void* q; const int* q_pos;
  const void* kc; const void* vc; int nc; int nc_cap; int r;
  const int* idx; int k;
  const void* kw; const void* vw; int ring; int W; float scale;
  void* o; float* lse;
  float* part_o; float* part_lse;  // split-KV partials (nsplit > 1)
  int T, H, D, nsplit;
  int real_kv;  // 1: each selected entry j stands for raw tokens jr .. jr+r-1, read from the ring
  // Bounded waits of the heads-in-M tensor-core kernel: the limit of every wait, and
  // a test hook that withholds one K-tile arrival in the first CTA so that the
  // waits expire (exercises the abort path; 0 in every product call).
  unsigned long long wait_ns;
  int test_drop_arrival;
};

// Key u of query t's list: u < n_comp -> compressed slot u, else window position.
// TPH threads per head (H = 256 / TPH), DPT channels per thread (D = TPH * DPT);
// thread `sub` of a head owns channels sub, sub + TPH, ... (conflict-free smem reads).
template <typename T, int TPH, int DPT>
__global__ void __launch_bounds__(kAttnThreads)
attn_ffma_kernel(AttnArgs a) {
  extern __shared__ float smem[];
  const int D = a.D, H = a.H;
  float* Ks = smem;                       // [kAttnTile][D]
  float* Vs = Ks + kAttnTile * D;         // [kAttnTile][D]
  __shared__ int s_valid[kAttnTile];

  const int i = blockIdx.x, b = blockIdx.y, split = blockIdx.z;
  const size_t row = (size_t)b * a.T + i;
  const int t = a.q_pos[row];
  const int vis = visible_entries(t, a.r, a.nc);
  const int n_comp = a.idx ? a.k : vis;
  const int w0 = t - a.W + 1 > 0 ? t - a.W + 1 : 0;
  const int n_win = a.W > 0 ? t - w0 + 1 : 0;
  const int n_keys = n_comp + n_win;
  const int per = (n_keys + a.nsplit - 1) / a.nsplit;
  const int u_beg = split * per;
  const int u_end = min(n_keys, u_beg + per);

  constexpr int tph = TPH;
  const int h = threadIdx.x / tph, sub = threadIdx.x % tph;
  const T* qrow = (const T*)a.q + (row * H + h) * D;
  float qv[DPT], acc[DPT];
#pragma unroll
  for (int e = 0; e < DPT; ++e) {
    qv[e] = to_f(qrow[sub + tph * e]) * a.scale;
    acc[e] = 0.f;
  }
  float m_run = -INFINITY, l_run = 0.f;
  const T* kcb = (const T*)a.kc + (size_t)b * a.nc_cap * D;
  const T* vcb = (const T*)a.vc + (size_t)b * a.nc_cap * D;
  const T* kwb = (const T*)a.kw + (size_t)b * a.ring * D;
  const T* vwb = (const T*)a.vw + (size_t)b * a.ring * D;
  const int* idxr = a.idx ? a.idx + row * a.k : nullptr;

  for (int u0 = u_beg; u0 < u_end; u0 += kAttnTile) {
    const int nt = min(kAttnTile, u_end - u0);
    // gather the tile: warp w loads keys w, w+8, ...
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int kk = warp; kk < kAttnTile; kk += kAttnThreads / 32) {
      const T* ksrc = nullptr;
      const T* vsrc = nullptr;
      if (kk < nt) {
        const int u = u0 + kk;
        if (u < n_comp) {
          const int j = idxr ? idxr[u] : u;
          if (j >= 0 && j < vis) {
            ksrc = kcb + (size_t)j * D;
            vsrc = vcb + (size_t)j * D;
          } else if (j >= 0 && lane == 0) {
            report(HYB_ERR_DEVICE_CHECK);
          }
        } else {
          const int s = w0 + (u - n_comp);
          ksrc = kwb + (size_t)(s % a.ring) * D;
          vsrc = vwb + (size_t)(s % a.ring) * D;
        }
      }
      if (lane == 0) s_valid[kk] = ksrc != nullptr;
      for (int c = lane; c < D; c += 32) {
        Ks[kk * D + c] = ksrc ? to_f(ksrc[c]) : 0.f;
        Vs[kk * D + c] = vsrc ? to_f(vsrc[c]) : 0.f;
      }
    }
    __syncthreads();
    float s[kAttnTile];
    float m_tile = -INFINITY;
#pragma unroll
    for (int kk = 0; kk < kAttnTile; ++kk) {
      float p = 0.f;
#pragma unroll
      for (int e = 0; e < DPT; ++e) p = fmaf(qv[e], Ks[kk * D + sub + tph * e], p);
#pragma unroll
      for (int o = 1; o < tph; o <<= 1) p += __shfl_xor_sync(0xffffffffu, p, o);
      s[kk] = s_valid[kk] ? p : -INFINITY;
      m_tile = fmaxf(m_tile, s[kk]);
    }
    const float m_new = fmaxf(m_run, m_tile);
    if (m_new != -INFINITY) {
      const float alpha = __expf(m_run - m_new);
      l_run *= alpha;
#pragma unroll
      for (int e = 0; e < DPT; ++e) acc[e] *= alpha;
#pragma unroll 4
      for (int kk = 0; kk < kAttnTile; ++kk) {
        const float p = __expf(s[kk] - m_new);
        l_run += p;
#pragma unroll
        for (int e = 0; e < DPT; ++e) acc[e] = fmaf(p, Vs[kk * D + sub + tph * e], acc[e]);
      }
      m_run = m_new;
    }
    __syncthreads();
  }

  const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
  const float lse = l_run > 0.f ? m_run + __logf(l_run) : -INFINITY;
  if (a.nsplit == 1) {
    T* orow = (T*)a.o + (row * H + h) * D;
#pragma unroll
    for (int e = 0; e < DPT; ++e) store_f(orow + sub + tph * e, acc[e] * inv);
    if (a.lse && sub == 0) a.lse[row * H + h] = lse;
  } else {
    const size_t prow = (row * a.nsplit + split) * H + h;
#pragma unroll
    for (int e = 0; e < DPT; ++e) a.part_o[prow * D + sub + tph * e] = acc[e] * inv;
    if (sub == 0) a.part_lse[prow] = lse;
  }
}

template <typename T, int TPH, int DPT>
cudaError_t launch_attn_ffma_cfg(const AttnArgs& a, int batch, cudaStream_t s) {
  const size_t smem = (size_t)2 * kAttnTile * a.D * 4;
  cudaError_t e = cudaFuncSetAttribute(attn_ffma_kernel<T, TPH, DPT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  attn_ffma_kernel<T, TPH, DPT><<<dim3(a.T, batch, a.nsplit), kAttnThreads, smem, s>>>(a);
  count_launch();
  return cudaGetLastError();
}

// Head/channel geometries built for the CUDA-core path (H = 256/TPH, D = TPH*DPT).
inline bool attn_ffma_supported(int H, int D) {
  return (H == 64 && (D == 128 || D == 64)) || (H == 8 && (D == 64 || D == 128)) ||
         (H == 16 && D == 128) || (H == 32 && D == 128);
}

template <typename T>
cudaError_t launch_attn_ffma(const AttnArgs& a, int batch, cudaStream_t s) {
  if (a.H == 64 && a.D == 128) return launch_attn_ffma_cfg<T, 4, 32>(a, batch, s);
  if (a.H == 64 && a.D == 64) return launch_attn_ffma_cfg<T, 4, 16>(a, batch, s);
  if (a.H == 8 && a.D == 64) return launch_attn_ffma_cfg<T, 32, 2>(a, batch, s);
  if (a.H == 8 && a.D == 128) return launch_attn_ffma_cfg<T, 32, 4>(a, batch, s);
  if (a.H == 16 && a.D == 128) return launch_attn_ffma_cfg<T, 16, 8>(a, batch, s);
  if (a.H == 32 && a.D == 128) return launch_attn_ffma_cfg<T, 8, 16>(a, batch, s);
  return cudaErrorInvalidValue;
}

// Combines the nsplit partial softmaxes of every (query, head).
template <typename T>
__global__ void attn_merge_kernel(AttnArgs a) {
  const size_t row = blockIdx.x;
  const int h = blockIdx.y, H = a.H, D = a.D, ns = a.nsplit;
  float mx = -INFINITY;
  for (int s = 0; s < ns; ++s) mx = fmaxf(mx, a.part_lse[(row * ns + s) * H + h]);
  float den = 0.f;
  for (int s = 0; s < ns; ++s) {
    const float l = a.part_lse[(row * ns + s) * H + h];
    den += l == -INFINITY ? 0.f : __expf(l - mx);
  }
  for (int c = threadIdx.x; c < D; c += blockDim.x) {
    float acc = 0.f;
    for (int s = 0; s < ns; ++s) {
      const float l = a.part_lse[(row * ns + s) * H + h];
      if (l != -INFINITY) acc += __expf(l - mx) * a.part_o[((row * ns + s) * H + h) * D + c];
    }
    store_f((T*)a.o + (row * H + h) * D + c, den > 0.f ? acc / den : 0.f);
  }
  if (a.lse && threadIdx.x == 0) a.lse[row * H + h] = den > 0.f ? mx + __logf(den) : -INFINITY;
}

}  // namespace hyb
