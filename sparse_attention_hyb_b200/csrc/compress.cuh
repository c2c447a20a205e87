// S1 — sequence-axis compression (HCA article, section "怎么压"): every entry is
// a softmax-weighted sum of the raw rows of its window, the weight of a token
// being softmax over the window of (its compression logit + the learnable bias
// of its position in the window).  CSA windows are 2r long at stride r, HCA
// windows r long without overlap.
//
// HBM-bound streaming pass.  The pooled sum over a window is defined part by
// part: parts of kPart consecutive window positions, each summed with fused
// multiply-adds in ascending position order, then combined in a fixed pairwise
// grouping (PartSum).  Every path computes exactly this, so the caches are bit-identical
// whichever kernel wrote them (the decode-step update included).
// Short windows (CSA, 8 tokens): one warp owns one entry; it computes the
// window's weights once (lanes over window positions) and pools K, V and the
// indexer keys with them (lanes over channels, 4 channels per lane, so a warp
// reads a whole 256-byte bf16 row per load).  Consecutive warps own consecutive
// entries, so the raw rows shared by two overlapping windows are read twice
// within a few hundred nanoseconds and the second read hits L2.
// Long windows (HCA, 128 tokens): one CTA per entry, one warp per part, so that
// the window's rows are read by several warps at once.
#pragma once
#include "common.cuh"

namespace hyb {

constexpr int kCompressWarps = 4;
constexpr int kMaxSpan = 256;
constexpr int kPart = 32;                      // window positions per partial sum
constexpr int kMaxParts = kMaxSpan / kPart;
constexpr int kPartsMaxC = 256;                // channels of the CTA-per-entry kernel
constexpr int kPartsEntries = 2048;            // entries below which it is used

// Window weights of one entry into w[0, span): softmax over the in-range tokens
// (position >= 0) of (logit + bias of the position in the window); z(s) returns
// the logit of token s.  One warp.
template <typename ZFn>
__device__ __forceinline__ void entry_weights(ZFn z, const float* __restrict__ bias, int start, int span, float* w,
                                              int lane) {
  float mx = -INFINITY;
  for (int p = lane; p < span; p += 32) {
    const int s = start + p;
    const float a = s >= 0 ? z(s) + bias[p] : -INFINITY;
    w[p] = a;
    mx = fmaxf(mx, a);
  }
  mx = warp_max(mx);
  float sum = 0.f;
  for (int p = lane; p < span; p += 32) {
    const float e = w[p] == -INFINITY ? 0.f : __expf(w[p] - mx);
    w[p] = e;
    sum += e;
  }
  sum = warp_sum(sum);
  const float inv = 1.f / sum;
  for (int p = lane; p < span; p += 32) w[p] *= inv;
  __syncwarp();
}

__device__ __forceinline__ float4 add4(float4 a, float4 b) { return make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w); }

// Partial sum of window positions [p0, p1) for the 4 channels at c: fused
// multiply-adds in ascending position order; positions of weight 0 (before the
// start of the sequence) are skipped.  NT tensors share the loop (one
// accumulator each, same arithmetic as NT = 1).
template <int NT, int UNROLL, typename RowFn>
__device__ __forceinline__ void pool_part(RowFn row, int c, int start, int p0, int p1, const float* w,
                                          float4 (&acc)[NT]) {
#pragma unroll
  for (int t = 0; t < NT; ++t) acc[t] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll UNROLL
  for (int p = p0; p < p1; ++p) {
    const float wp = w[p];
    if (wp == 0.f) continue;
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      const float4 v = load4(row(t, start + p) + c);
      acc[t].x = fmaf(wp, v.x, acc[t].x);
      acc[t].y = fmaf(wp, v.y, acc[t].y);
      acc[t].z = fmaf(wp, v.z, acc[t].z);
      acc[t].w = fmaf(wp, v.w, acc[t].w);
    }
  }
}

// Sum of a window's parts in a fixed pairwise grouping, built part by part like a
// binary counter: p0 + p1 -> s01, p2 + p3 -> s23, s01 + s23 -> s0123, ...; what is
// left pending at the end is added from the most recent part upward (with seven
// parts: s0123 + (s45 + p6)).  Registers only; every path uses this object.
struct PartSum {
  float4 l0, l1, l2, l3;   // pending sums of 1, 2, 4 and 8 parts
  unsigned pend = 0;
  __device__ __forceinline__ void add(float4 v) {
    if (!(pend & 1u)) { l0 = v; pend |= 1u; return; }
    v = add4(l0, v);
    if (!(pend & 2u)) { l1 = v; pend = (pend & ~1u) | 2u; return; }
    v = add4(l1, v);
    if (!(pend & 4u)) { l2 = v; pend = (pend & ~3u) | 4u; return; }
    v = add4(l2, v);
    l3 = v;
    pend = (pend & ~7u) | 8u;
  }
  __device__ __forceinline__ float4 total() const {
    float4 r = make_float4(0.f, 0.f, 0.f, 0.f);
    bool have = false;
    if (pend & 1u) { r = l0; have = true; }
    if (pend & 2u) { r = have ? add4(l1, r) : l1; have = true; }
    if (pend & 4u) { r = have ? add4(l2, r) : l2; have = true; }
    if (pend & 8u) { r = have ? add4(l3, r) : l3; }
    return r;
  }
};

__host__ __device__ __forceinline__ int n_parts(int span) { return (span + kPart - 1) / kPart; }

// out[c] = sum_p w[p] * row(start + p)[c] over C channels (4 per lane) for a window
// of one part (span <= kPart): one chain of multiply-adds.  row(s) returns the
// address of token s's row.  One warp.
template <typename T, typename RowFn>
__device__ __forceinline__ void pool_entry_short(RowFn row, T* __restrict__ out, int C, int start, int span,
                                                 const float* w, int lane) {
  for (int c = lane * 4; c < C; c += 128) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
    for (int p = 0; p < span; ++p) {
      const float wp = w[p];
      if (wp == 0.f) continue;  // token before the start of the sequence
      const float4 v = load4(row(start + p) + c);
      acc.x = fmaf(wp, v.x, acc.x);
      acc.y = fmaf(wp, v.y, acc.y);
      acc.z = fmaf(wp, v.z, acc.z);
      acc.w = fmaf(wp, v.w, acc.w);
    }
    store4(out + c, acc);
  }
}

// The same for a window of several parts: each part's chain, then PartSum.  One warp.
template <typename T, typename RowFn>
__device__ __forceinline__ void pool_entry_long(RowFn row, T* __restrict__ out, int C, int start, int span,
                                                const float* w, int lane) {
  const int np = n_parts(span);
  auto row1 = [row](int, int s) { return row(s); };
  for (int c = lane * 4; c < C; c += 128) {
    PartSum ps;
#pragma unroll 1
    for (int q = 0; q < np; ++q) {
      float4 part[1];
      pool_part<1, 8>(row1, c, start, q * kPart, min(span, (q + 1) * kPart), w, part);
      ps.add(part[0]);
    }
    store4(out + c, ps.total());
  }
}

template <typename T, typename RowFn>
__device__ __forceinline__ void pool_entry(RowFn row, T* __restrict__ out, int C, int start, int span, const float* w,
                                           int lane) {
  if (n_parts(span) == 1) pool_entry_short(row, out, C, start, span, w, lane);
  else pool_entry_long(row, out, C, start, span, w, lane);
}

// Long windows: one CTA per entry; warp q computes the window's weights itself and
// sums part q of the window for K and V (and the indexer keys) in one loop, then
// the threads combine the parts channel group by channel group.
template <typename T>
__global__ void __launch_bounds__(kMaxParts * 32)
compress_parts_kernel(const T* __restrict__ xk, const T* __restrict__ xv, const T* __restrict__ xi,
                      const float* __restrict__ logits, const float* __restrict__ bias,
                      T* __restrict__ kc, T* __restrict__ vc, T* __restrict__ ic,
                      int L, int D, int dI, int r, int overlap, int j_begin, int nc_cap) {
  __shared__ float w[kMaxParts][kMaxSpan];
  __shared__ float4 part[3][kMaxParts][kPartsMaxC / 4];
  const int b = blockIdx.y, j = j_begin + blockIdx.x;
  const int q = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int span = overlap ? 2 * r : r, np = n_parts(span);
  const int start = overlap ? (j - 1) * r : j * r;
  const float* zb = logits + (size_t)b * L;
  entry_weights([&](int s) { return zb[s]; }, bias, start, span, w[q], lane);
  const size_t row0 = (size_t)b * L;
  const int p0 = q * kPart, p1 = min(span, (q + 1) * kPart);
  const T* k0 = xk + row0 * D;
  const T* v0 = xv + row0 * D;
  for (int c = lane * 4; c < D; c += 128) {
    float4 acc[2];
    pool_part<2, 8>([=](int t, int s) { return (t == 0 ? k0 : v0) + (size_t)s * D; }, c, start, p0, p1, w[q], acc);
    part[0][q][c / 4] = acc[0];
    part[1][q][c / 4] = acc[1];
  }
  if (xi != nullptr)
    for (int c = lane * 4; c < dI; c += 128) {
      float4 acc[1];
      pool_part<1, 8>([=](int, int s) { return xi + (row0 + s) * dI; }, c, start, p0, p1, w[q], acc);
      part[2][q][c / 4] = acc[0];
    }
  __syncthreads();
  const size_t out0 = (size_t)b * nc_cap + j;
  for (int g = threadIdx.x; g < D / 4; g += blockDim.x)
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      PartSum ps;
      for (int i = 0; i < np; ++i) ps.add(part[t][i][g]);
      store4((t == 0 ? kc : vc) + out0 * D + 4 * g, ps.total());
    }
  if (xi != nullptr)
    for (int g = threadIdx.x; g < dI / 4; g += blockDim.x) {
      PartSum ps;
      for (int i = 0; i < np; ++i) ps.add(part[2][i][g]);
      store4(ic + out0 * dI + 4 * g, ps.total());
    }
}

// One warp per entry; LONG: windows of several parts (span > kPart).
template <typename T, bool LONG>
__global__ void __launch_bounds__(kCompressWarps * 32)
compress_kernel(const T* __restrict__ xk, const T* __restrict__ xv, const T* __restrict__ xi,
                const float* __restrict__ logits, const float* __restrict__ bias,
                T* __restrict__ kc, T* __restrict__ vc, T* __restrict__ ic,
                int L, int D, int dI, int r, int overlap, int j_begin, int j_end, int nc_cap) {
  __shared__ float wts[kCompressWarps][kMaxSpan];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.y;
  const int j = j_begin + blockIdx.x * kCompressWarps + warp;
  if (j >= j_end) return;
  const int span = overlap ? 2 * r : r;
  const int start = overlap ? (j - 1) * r : j * r;
  const float* zb = logits + (size_t)b * L;
  float* w = wts[warp];
  entry_weights([&](int s) { return zb[s]; }, bias, start, span, w, lane);
  const size_t row0 = (size_t)b * L;
  const size_t out0 = (size_t)b * nc_cap + j;
  if constexpr (LONG) {
    // K and V share each part's loop (twice the loads in flight); each keeps its own
    // chain, so the arithmetic is that of pool_entry_long
    const int np = n_parts(span);
    const T* k0 = xk + row0 * D;
    const T* v0 = xv + row0 * D;
    for (int c = lane * 4; c < D; c += 128) {
      PartSum pk, pv;
#pragma unroll 1
      for (int q = 0; q < np; ++q) {
        float4 acc[2];
        pool_part<2, 8>([=](int t, int s) { return (t == 0 ? k0 : v0) + (size_t)s * D; }, c, start, q * kPart,
                        min(span, (q + 1) * kPart), w, acc);
        pk.add(acc[0]);
        pv.add(acc[1]);
      }
      store4(kc + out0 * D + c, pk.total());
      store4(vc + out0 * D + c, pv.total());
    }
    if (xi != nullptr)
      pool_entry_long([&](int s) { return xi + (row0 + s) * dI; }, ic + out0 * dI, dI, start, span, w, lane);
  } else if (xi != nullptr && dI == D && D <= 128) {
    // K, V and the indexer keys of the same width share one loop over the window
    // (one weight read and one skip test per position for the three; each keeps its
    // own chain of multiply-adds, the arithmetic of pool_entry_short)
    const int c = lane * 4;
    if (c < D) {
      float4 a0 = make_float4(0.f, 0.f, 0.f, 0.f), a1 = a0, a2 = a0;
      const T* k0 = xk + row0 * D + c;
      const T* v0 = xv + row0 * D + c;
      const T* i0 = xi + row0 * D + c;
#pragma unroll 4
      for (int p = 0; p < span; ++p) {
        const float wp = w[p];
        if (wp == 0.f) continue;  // token before the start of the sequence
        const size_t o = (size_t)(start + p) * D;
        const float4 x0 = load4(k0 + o), x1 = load4(v0 + o), x2 = load4(i0 + o);
        a0.x = fmaf(wp, x0.x, a0.x); a0.y = fmaf(wp, x0.y, a0.y); a0.z = fmaf(wp, x0.z, a0.z); a0.w = fmaf(wp, x0.w, a0.w);
        a1.x = fmaf(wp, x1.x, a1.x); a1.y = fmaf(wp, x1.y, a1.y); a1.z = fmaf(wp, x1.z, a1.z); a1.w = fmaf(wp, x1.w, a1.w);
        a2.x = fmaf(wp, x2.x, a2.x); a2.y = fmaf(wp, x2.y, a2.y); a2.z = fmaf(wp, x2.z, a2.z); a2.w = fmaf(wp, x2.w, a2.w);
      }
      store4(kc + out0 * D + c, a0);
      store4(vc + out0 * D + c, a1);
      store4(ic + out0 * D + c, a2);
    }
  } else {
    pool_entry_short([&](int s) { return xk + (row0 + s) * D; }, kc + out0 * D, D, start, span, w, lane);
    pool_entry_short([&](int s) { return xv + (row0 + s) * D; }, vc + out0 * D, D, start, span, w, lane);
    if (xi != nullptr)
      pool_entry_short([&](int s) { return xi + (row0 + s) * dI; }, ic + out0 * dI, dI, start, span, w, lane);
  }
}

// S1 with per-channel compression weights: channel c of entry j pools its window
// with w[., c] = softmax over the in-range tokens of (z[s, c] + bias[p, c]).  K and
// V share the logits z_kv [L, D] and bias_kv [span, D]; the indexer keys have
// their own z_i [L, dI], bias_i [span, dI].  One warp per entry; a lane owns 4
// channels and computes their softmax itself (no cross-lane reduction): one pass
// over the window's logits for the maximum, one for the weights and the pooling.
template <typename T>
__device__ __forceinline__ void pool_entry_pc(const T* __restrict__ x0, const T* __restrict__ x1,
                                              const float* __restrict__ z, const float* __restrict__ bias,
                                              T* __restrict__ o0, T* __restrict__ o1, int C, int start, int span,
                                              int lane) {
  for (int c = lane * 4; c < C; c += 128) {
    float4 mx = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
    for (int p = 0; p < span; ++p) {
      const int s = start + p;
      if (s < 0) continue;
      const float4 zz = *reinterpret_cast<const float4*>(z + (size_t)s * C + c);
      const float4 bb = *reinterpret_cast<const float4*>(bias + (size_t)p * C + c);
      mx.x = fmaxf(mx.x, zz.x + bb.x); mx.y = fmaxf(mx.y, zz.y + bb.y);
      mx.z = fmaxf(mx.z, zz.z + bb.z); mx.w = fmaxf(mx.w, zz.w + bb.w);
    }
    float4 sum = make_float4(0.f, 0.f, 0.f, 0.f), a0 = sum, a1 = sum;
    for (int p = 0; p < span; ++p) {
      const int s = start + p;
      if (s < 0) continue;
      const float4 zz = *reinterpret_cast<const float4*>(z + (size_t)s * C + c);
      const float4 bb = *reinterpret_cast<const float4*>(bias + (size_t)p * C + c);
      const float4 e = make_float4(__expf(zz.x + bb.x - mx.x), __expf(zz.y + bb.y - mx.y), __expf(zz.z + bb.z - mx.z),
                                   __expf(zz.w + bb.w - mx.w));
      sum.x += e.x; sum.y += e.y; sum.z += e.z; sum.w += e.w;
      const float4 v0 = load4(x0 + (size_t)s * C + c);
      a0.x = fmaf(e.x, v0.x, a0.x); a0.y = fmaf(e.y, v0.y, a0.y);
      a0.z = fmaf(e.z, v0.z, a0.z); a0.w = fmaf(e.w, v0.w, a0.w);
      if (x1 != nullptr) {
        const float4 v1 = load4(x1 + (size_t)s * C + c);
        a1.x = fmaf(e.x, v1.x, a1.x); a1.y = fmaf(e.y, v1.y, a1.y);
        a1.z = fmaf(e.z, v1.z, a1.z); a1.w = fmaf(e.w, v1.w, a1.w);
      }
    }
    store4(o0 + c, make_float4(a0.x / sum.x, a0.y / sum.y, a0.z / sum.z, a0.w / sum.w));
    if (x1 != nullptr) store4(o1 + c, make_float4(a1.x / sum.x, a1.y / sum.y, a1.z / sum.z, a1.w / sum.w));
  }
}

template <typename T>
__global__ void __launch_bounds__(kCompressWarps * 32)
compress_pc_kernel(const T* __restrict__ xk, const T* __restrict__ xv, const T* __restrict__ xi,
                   const float* __restrict__ z_kv, const float* __restrict__ bias_kv, const float* __restrict__ z_i,
                   const float* __restrict__ bias_i, T* __restrict__ kc, T* __restrict__ vc, T* __restrict__ ic,
                   int L, int D, int dI, int r, int overlap, int j_begin, int j_end, int nc_cap) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.y;
  const int j = j_begin + blockIdx.x * kCompressWarps + warp;
  if (j >= j_end) return;
  const int span = overlap ? 2 * r : r;
  const int start = overlap ? (j - 1) * r : j * r;
  const size_t row0 = (size_t)b * L, out0 = (size_t)b * nc_cap + j;
  pool_entry_pc(xk + row0 * D, xv + row0 * D, z_kv + row0 * D, bias_kv, kc + out0 * D, vc + out0 * D, D, start, span,
                lane);
  if (xi != nullptr)
    pool_entry_pc<T>(xi + row0 * dI, nullptr, z_i + row0 * dI, bias_i, ic + out0 * dI, nullptr, dI, start, span, lane);
}

template <typename T>
cudaError_t launch_compress(int batch, int L, int D, int dI, const void* xk, const void* xv,
                            const void* xi, const float* logits, const float* bias, int r,
                            int overlap, int j_begin, int j_end, void* kc, void* vc, void* ic,
                            int nc_cap, cudaStream_t stream) {
  const int n = j_end - j_begin;
  if (n <= 0 || batch <= 0) return cudaSuccess;
  const int span = overlap ? 2 * r : r;
  // long windows with too few entries to give every SM several warps (a warp per
  // entry reads its window part after part): one CTA per entry, one warp per part
  if (n_parts(span) > 1 && (long long)n * batch < kPartsEntries && D <= kPartsMaxC &&
      (xi == nullptr || dI <= kPartsMaxC)) {
    compress_parts_kernel<T><<<dim3(n, batch), n_parts(span) * 32, 0, stream>>>(
        (const T*)xk, (const T*)xv, (const T*)xi, logits, bias, (T*)kc, (T*)vc, (T*)ic, L, D, dI, r, overlap,
        j_begin, nc_cap);
    count_launch();
    return cudaGetLastError();
  }
  dim3 grid((n + kCompressWarps - 1) / kCompressWarps, batch);
  auto kern = n_parts(span) > 1 ? compress_kernel<T, true> : compress_kernel<T, false>;
  kern<<<grid, kCompressWarps * 32, 0, stream>>>((const T*)xk, (const T*)xv, (const T*)xi, logits, bias, (T*)kc,
                                                 (T*)vc, (T*)ic, L, D, dI, r, overlap, j_begin, j_end, nc_cap);
  count_launch();
  return cudaGetLastError();
}

// Decode-step state update, fused (one warp per sequence).  The new token t =
// pos[b] goes to slot t mod ring of the window rings (K, V, and the indexer key
// and logit, which compression needs); when t closes a CSA window ((t + 1) is a
// multiple of r) entry (t + 1) / r - 1 is pooled from the rings with the same
// device functions, hence the same arithmetic, as compress_kernel; likewise an
// HCA entry; and when the CSA entry completes a block of `block` entries, that
// block's representative is recomputed as block_reps_kernel does.  Every window
// lies inside the rings (span <= ring is checked on the host).
template <typename T>
__global__ void __launch_bounds__(32)
decode_append_kernel(const T* __restrict__ xk_new, const T* __restrict__ xv_new, const T* __restrict__ xi_new,
                     const float* __restrict__ z_new, const int* __restrict__ pos, T* kw, T* vw, T* iw, float* zw,
                     int ring, int D, int dI, const float* __restrict__ bias_c, int r_c, int overlap_c, T* kc, T* vc,
                     T* ic, int nc_cap, const float* __restrict__ bias_h, int r_h, T* kch, T* vch, int nch_cap,
                     int block, T* reps, int nb_cap) {
  __shared__ float w[kMaxSpan];
  const int b = blockIdx.x, lane = threadIdx.x;
  const int t = pos[b];
  if (t < 0) {
    if (lane == 0) report(HYB_ERR_DEVICE_CHECK);
    return;
  }
  const size_t rb = (size_t)b * ring;
  const size_t slot = rb + t % ring;
  for (int c = lane * 4; c < D; c += 128) {
    store4(kw + slot * D + c, load4(xk_new + (size_t)b * D + c));
    store4(vw + slot * D + c, load4(xv_new + (size_t)b * D + c));
  }
  if (iw != nullptr)
    for (int c = lane * 4; c < dI; c += 128) store4(iw + slot * dI + c, load4(xi_new + (size_t)b * dI + c));
  if (lane == 0) zw[slot] = z_new[b];
  __syncwarp();
  auto zr = [&](int s) { return zw[rb + s % ring]; };
  if (bias_c != nullptr && (t + 1) % r_c == 0) {
    const int j = (t + 1) / r_c - 1;
    if (j >= nc_cap) {
      if (lane == 0) report(HYB_ERR_DEVICE_CHECK);
    } else {
      const int span = overlap_c ? 2 * r_c : r_c, start = overlap_c ? (j - 1) * r_c : j * r_c;
      entry_weights(zr, bias_c, start, span, w, lane);
      const size_t o = (size_t)b * nc_cap + j;
      pool_entry([&](int s) { return kw + (rb + s % ring) * D; }, kc + o * D, D, start, span, w, lane);
      pool_entry([&](int s) { return vw + (rb + s % ring) * D; }, vc + o * D, D, start, span, w, lane);
      if (iw != nullptr && ic != nullptr)
        pool_entry([&](int s) { return iw + (rb + s % ring) * dI; }, ic + o * dI, dI, start, span, w, lane);
      __syncwarp();
      if (reps != nullptr && ic != nullptr && block > 0 && (j + 1) % block == 0 && (j + 1) / block - 1 < nb_cap) {
        const int g = (j + 1) / block - 1;
        const T* src = ic + ((size_t)b * nc_cap + (size_t)g * block) * dI;
        const float inv = 1.f / (float)block;
        for (int c = lane * 4; c < dI; c += 128) {
          float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
          for (int e = 0; e < block; ++e) {
            const float4 v = load4(src + (size_t)e * dI + c);
            acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
          }
          acc.x *= inv; acc.y *= inv; acc.z *= inv; acc.w *= inv;
          store4(reps + ((size_t)b * nb_cap + g) * dI + c, acc);
        }
      }
    }
  }
  __syncwarp();
  if (bias_h != nullptr && (t + 1) % r_h == 0) {
    const int j = (t + 1) / r_h - 1;
    if (j >= nch_cap) {
      if (lane == 0) report(HYB_ERR_DEVICE_CHECK);
    } else {
      const int start = j * r_h;
      entry_weights(zr, bias_h, start, r_h, w, lane);
      const size_t o = (size_t)b * nch_cap + j;
      pool_entry([&](int s) { return kw + (rb + s % ring) * D; }, kch + o * D, D, start, r_h, w, lane);
      pool_entry([&](int s) { return vw + (rb + s % ring) * D; }, vch + o * D, D, start, r_h, w, lane);
    }
  }
}

// HISA block representatives: the mean of the indexer keys of a full block.
template <typename T>
__global__ void block_reps_kernel(const T* __restrict__ ic, T* __restrict__ reps, int dI,
                                  int nc_cap, int block, int g_begin, int nb_cap) {
  const int g = g_begin + blockIdx.x, b = blockIdx.y;
  const T* src = ic + ((size_t)b * nc_cap + (size_t)g * block) * dI;
  const float inv = 1.f / (float)block;
  for (int c = threadIdx.x * 4; c < dI; c += blockDim.x * 4) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int e = 0; e < block; ++e) {
      const float4 v = load4(src + (size_t)e * dI + c);
      acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
    }
    acc.x *= inv; acc.y *= inv; acc.z *= inv; acc.w *= inv;
    store4(reps + ((size_t)b * nb_cap + g) * dI + c, acc);
  }
}

template <typename T>
cudaError_t launch_block_reps(int batch, int dI, const void* ic, int nc_cap, int block, int g_begin,
                              int g_end, void* reps, int nb_cap, cudaStream_t stream) {
  const int n = g_end - g_begin;
  if (n <= 0 || batch <= 0) return cudaSuccess;
  const int threads = dI / 4 < 32 ? 32 : (dI / 4 > 256 ? 256 : dI / 4);
  block_reps_kernel<T><<<dim3(n, batch), threads, 0, stream>>>((const T*)ic, (T*)reps, dI, nc_cap,
                                                               block, g_begin, nb_cap);
  count_launch();
  return cudaGetLastError();
}

}  // namespace hyb
