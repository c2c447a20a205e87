// S3 + S4 on the 5th-generation tensor cores with the heads in the M dimension:
// shared-KV (MQA) attention of the 64 query heads of one query over its selected
// (CSA) or all visible (HCA) compressed entries plus the sliding window, under
// one joint softmax (HCA article, section "怎么压"; trdm.cn 2.1).
//
// Per query and 128-key tile j (M = 64 heads, one query at a time):
//   S_j  = Q . K_j^T             tcgen05 M=64, N=128 keys, K=128 (A = Q, B = K_j, both shared memory)
//   P_j  = exp2(S_j*c - m)       written to a P buffer in tensor memory as bf16
//   O   += P_j . V_j             tcgen05 M=64, N=128 (head dim), K=128 keys, A = P_j from tensor memory
// An M=64 accumulator occupies lanes 0-15 of each 32-lane quadrant of tensor
// memory; a softmax thread owns 32 keys of one head row (the 16x32bx2 access
// shape: threads l and l + 16 of a warp hold the same row), so the row maximum and
// sum need one shuffle and one exchange with the partner warp of the quadrant.
// Probabilities never leave tensor memory.
//
// Roles (18 warps, one persistent CTA per SM):
//   warps 0-7   softmax and epilogue: warps q and q+4 read TMEM lane quadrant q
//               and split each tile's keys (and O's head-dim columns) in halves;
//   warp 8      TMEM owner; lane 0 issues every MMA as two streams scheduled by
//               readiness (S of later tiles while the softmax works, O updates as
//               probabilities arrive), from precomputed descriptors;
//   warp 9      Q tiles (2-D TMA into two slots, the next queries' tiles and
//               indexer rows prefetched into L2);
//   warps 10-13 K tiles, warps 14-17 V tiles: gathered rows are copied with
//               16-byte cp.async, 16 lanes per 256-byte row (whole cache lines per
//               copy instruction), in the 128-byte swizzle the MMA expects; a tile
//               of 128 consecutive valid rows (window, or a full tile of a dense
//               compressed range) is one 2-D TMA box per 64-column half.  K
//               producers also publish the tile's validity mask (ballot).
// Ring depths: 2 Q, 3 K, 3 V tiles in shared memory (224 KB); in tensor memory
// three S buffers and one O accumulator (512 columns).  P_G (bf16 pairs) is
// written over the first half of S_G's buffer once both softmax warps of a
// quadrant have loaded it (their exchange of the row maximum orders the two), so
// the softmax never waits for an O update before storing P; S_{G+3} waits for
// the O update of tile G, which frees the buffer.
//
// Softmax: the running maximum m (base-2 units) only moves when a tile exceeds it
// by more than 8, and then O in tensor memory and the row sum are rescaled after
// the previous O update completed; otherwise probabilities are taken against the
// stale maximum (they stay below 2^8).  Masked keys (indexer padding, entries
// outside the visible range, window positions past the query) get probability 0
// and their rows are zero-filled without a global read.  A query's epilogue
// (o = O / l, lse) runs one tile late, inside the next query's first tile just
// before its P store, so the softmax does not wait for the query's last O update.
//
// A work item is a query, or in split-KV decode a tile-aligned slice of its keys
// whose partial (o, lse) attn_merge combines.  Every wait is bounded (AttnArgs::
// wait_ns of %globaltimer, 1 s in product calls): on expiry the CTA raises its
// abort flag, reports HYB_ERR_TIMEOUT, every role leaves its loop, the MMAs issued
// so far complete and the tensor memory is freed.
#pragma once
#include "attn.cuh"
#include "attn_tc.cuh"
#include "common.cuh"
#include "sm100.cuh"

namespace hyb {

namespace attn_hm {

using attn_tc::Item;
using attn_tc::KeyList;
using attn_tc::Maps;
using attn_tc::div_fast;

constexpr int kH = 64, kD = 128, kTile = 128;
constexpr int kQSt = 2, kKSt = 3, kVSt = 3, kSBuf = 3, kMSt = 4;
constexpr int kSmxWarps = 8, kMmaWarp = 8, kQWarp = 9, kKWarp0 = 10, kVWarp0 = 14;
constexpr int kThreads = 18 * 32;
constexpr int kQBytes = kH * kD * 2;      // 16 KB: two 64-column halves of 64 rows x 128 B
constexpr int kKVBytes = kTile * kD * 2;  // 32 KB: two 64-column halves of 128 rows x 128 B
constexpr int kSmem = kQSt * kQBytes + (kKSt + kVSt) * kKVBytes + 1024;
static_assert(kMSt > kKSt, "the mask ring must not hold back the K producers");
constexpr uint32_t kSCols = 128;              // one S buffer: 128 fp32 columns (three: 0 .. 383);
                                              // P over its first 64 columns
constexpr uint32_t kOCol = kSBuf * kSCols;    // O accumulator: columns 384 .. 511
constexpr float kRescaleThreshold = 8.f;

// ------------------------------------------------------------ tensor-memory access
// 16 lanes (quadrant base + 0..15) x 32 columns, two halves: thread l < 16 gets lane
// l, columns [c, c+32); thread l + 16 gets lane l, columns [c+32, c+64).
__device__ __forceinline__ void ld16x2_x32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x32bx2.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32], 32;"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
        "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
        "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr));
}
// Same shape with 16 columns per half: thread l < 16 gets columns [c, c+16), l + 16 [c+16, c+32).
__device__ __forceinline__ void ld16x2_x16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x32bx2.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16], 16;"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr));
}
__device__ __forceinline__ void st16x2_x16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x32bx2.x16.b32 [%0], 16, "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
      "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}
__device__ __forceinline__ void st16x2_x8(uint32_t taddr, const uint32_t (&v)[8]) {
  asm volatile("tcgen05.st.sync.aligned.16x32bx2.x8.b32 [%0], 8, {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(v[0]),
               "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// D[tmem] (+)= A[tmem] * B[smem], kind::f16 (A: bf16 in tensor memory, K-major).
__device__ __forceinline__ void mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
      ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Prefetch of `bytes` (a multiple of 16) from a 16-byte aligned global address into L2.
__device__ __forceinline__ void bulk_prefetch_l2(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t full_par(uint32_t n, int nst) { return (n / nst) & 1u; }
__device__ __forceinline__ uint32_t empty_par(uint32_t n, int nst) { return ((n / nst) & 1u) ^ 1u; }

// Source of key row `rr` of tile `tile` of a query's key list: the global row of
// K/V (compressed cache or window ring), or -1 for a masked key; -2 for an
// indexer entry outside the visible range (masked and reported).
__device__ __forceinline__ int key_row(const AttnArgs& a, const KeyList& kl, int b, int tile, int rr) {
  if (tile < kl.comp_tiles) {
    const int u = tile * kTile + rr;
    if (u >= kl.n_comp) return -1;
    const int e = a.idx ? __ldg(a.idx + (size_t)kl.row * a.k + u) : u;
    if (e < 0) return -1;
    if (e >= kl.vis) return -2;
    return b * a.nc_cap + e;
  }
  const int u = (tile - kl.comp_tiles) * kTile + rr;
  if (u >= kl.n_win) return -1;
  const int s = kl.w0_slot + u;   // < 2 ring: u < n_win <= W <= ring
  return b * a.ring + (s >= a.ring ? s - a.ring : s);
}

// First global row of a tile whose 128 keys are consecutive valid rows (one TMA box
// per half), else -1.
__device__ __forceinline__ int tile_box_row(const AttnArgs& a, const KeyList& kl, int b, int tile) {
  if (tile < kl.comp_tiles) {
    if (a.idx || (tile + 1) * kTile > kl.n_comp) return -1;
    return b * a.nc_cap + tile * kTile;
  }
  const int u0 = (tile - kl.comp_tiles) * kTile;
  if (u0 + kTile > kl.n_win) return -1;
  int s0 = kl.w0_slot + u0;
  if (s0 >= a.ring) s0 -= a.ring;
  return s0 + kTile <= a.ring ? b * a.ring + s0 : -1;
}

__global__ void __launch_bounds__(kThreads, 1)
attn_hm_kernel(const __grid_constant__ Maps maps, AttnArgs a, int n_items) {
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + kQSt * kQBytes;
  uint8_t* sV = sK + kKSt * kKVBytes;

  __shared__ uint64_t q_full[kQSt], q_empty[kQSt], k_full[kKSt], k_empty[kKSt], v_full[kVSt], v_empty[kVSt];
  __shared__ uint64_t s_full[kSBuf], p_full[kSBuf], o_bar[kSBuf], o_free, m_full[kMSt], m_empty[kMSt];
  __shared__ uint64_t mma_done;
  __shared__ __align__(16) uint32_t mask[kMSt][4];
  __shared__ uint64_t xbar[4][2], lbar[4];     // softmax pair exchanges (per lane quadrant)
  __shared__ float red[2][2][4][16], redl[2][4][16];
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    abort_flag = 0;
    for (int s = 0; s < kQSt; ++s) { mbar_init(&q_full[s], 1); mbar_init(&q_empty[s], 1); }
    for (int s = 0; s < kKSt; ++s) { mbar_init(&k_full[s], 128); mbar_init(&k_empty[s], 1); }
    for (int s = 0; s < kVSt; ++s) { mbar_init(&v_full[s], 128); mbar_init(&v_empty[s], 1); }
    for (int s = 0; s < kSBuf; ++s) { mbar_init(&s_full[s], 1); mbar_init(&p_full[s], kSmxWarps); }
    for (int s = 0; s < kSBuf; ++s) mbar_init(&o_bar[s], 1);
    mbar_init(&o_free, kSmxWarps);
    for (int s = 0; s < kMSt; ++s) { mbar_init(&m_full[s], 4); mbar_init(&m_empty[s], kSmxWarps); }
    for (int s = 0; s < 4; ++s) { mbar_init(&xbar[s][0], 2); mbar_init(&xbar[s][1], 2); mbar_init(&lbar[s], 2); }
    mbar_init(&mma_done, 1);
    fence_mbar_init();
  }
  if (warp == kMmaWarp) tmem_alloc(&tmem_base, 512);
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = tmem_base;
  const unsigned long long lim = a.wait_ns;   // limit of every wait

  if (warp < kSmxWarps) {
    // ======================================================== softmax + epilogue
    // Warps q and q + 4 share TMEM lane quadrant q (heads 16q .. 16q+15): warp q takes
    // keys 0..63 of each tile and head-dim columns 0..63 of O, warp q + 4 the other
    // halves; the row maximum and the row sum are exchanged between the pair.
    const int q4 = warp & 3, hw = warp >> 2;
    const int hi = lane >> 4;
    const int r16 = lane & 15;
    const int h = q4 * 16 + r16;              // head row
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const float c2 = a.scale * 1.4426950408889634f;   // scale * log2(e)
    uint32_t G = 0, n_ep = 0;                 // tiles processed; epilogues done
    bool ok = true;
    // waits until the O update of tile g completed; `ok` stays warp-uniform (the
    // tensor-memory accesses that follow are warp-collective)
    auto wait_o = [&](uint32_t g) {
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&o_bar[g % kSBuf], full_par(g, kSBuf), &abort_flag, lim));
    };
    // one value per head row shared with the partner warp through `slot`, ordered by
    // the pair's barrier `bar` (phase `par`); returns the partner's value
    auto exchange = [&](float v, float* slot_mine, const float* slot_other, uint64_t* bar, uint32_t par) {
      if (hi == 0) slot_mine[r16] = v;
      __syncwarp();
      if (lane == 0) mbar_arrive(bar);
      ok = __all_sync(0xffffffffu, mbar_wait(bar, par, &abort_flag, lim)) && ok;
      return slot_other[r16];
    };
    // ---- epilogue of an item: its last O update complete, then o = O / l (deferred by one tile)
    bool pend = false, e_final = true;
    size_t e_prow = 0;
    float e_m = 0.f, e_l = 0.f;
    uint32_t e_G = 0;
    auto epilogue = [&]() {
      pend = false;
      const float l = e_l, m_use = e_m;
      const size_t prow = e_prow;
      const bool final_out = e_final;
      wait_o(e_G);
      if (!ok) return;
      fence_after_sync();
      float lt = l + __shfl_xor_sync(0xffffffffu, l, 16);
      lt += exchange(lt, redl[hw][q4], redl[hw ^ 1][q4], &lbar[q4], n_ep & 1u);
      ++n_ep;
      if (!ok) return;
      const float inv = lt > 0.f ? 1.f / lt : 0.f;
      uint32_t ov[2][16];
#pragma unroll
      for (int c = 0; c < 2; ++c) ld16x2_x16(lane_addr + kOCol + 64 * hw + 32 * c, ov[c]);
      tmem_wait_ld();
      fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&o_free);   // the accumulator may be overwritten by the next item
      if (hw == 0 && hi == 0) {
        const float lse = lt > 0.f ? m_use * 0.6931471805599453f + logf(lt) : -INFINITY;
        if (final_out) { if (a.lse) a.lse[prow + h] = lse; }
        else a.part_lse[prow + h] = lse;
      }
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int d0 = 64 * hw + 32 * c + 16 * hi;
        if (final_out) {
          uint32_t pk[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            __nv_bfloat162 x2 = __floats2bfloat162_rn(__uint_as_float(ov[c][2 * i]) * inv,
                                                      __uint_as_float(ov[c][2 * i + 1]) * inv);
            pk[i] = *reinterpret_cast<uint32_t*>(&x2);
          }
          uint4* dst = reinterpret_cast<uint4*>(static_cast<bf16*>(a.o) + (prow + h) * kD + d0);
          dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        } else {
          float4* dst = reinterpret_cast<float4*>(a.part_o + (prow + h) * kD + d0);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            dst[i] = make_float4(__uint_as_float(ov[c][4 * i]) * inv, __uint_as_float(ov[c][4 * i + 1]) * inv,
                                 __uint_as_float(ov[c][4 * i + 2]) * inv, __uint_as_float(ov[c][4 * i + 3]) * inv);
        }
      }
    };
    for (int w = blockIdx.x; w < n_items && ok; w += gridDim.x) {
      Item it;
      it.init(a, w, false);
      const bool final_out = a.nsplit == 1;
      const size_t prow = final_out ? (size_t)it.kl.row * kH : ((size_t)it.kl.row * a.nsplit + it.split) * kH;
      if (it.n_tiles() == 0) {   // no key in this slice (split-KV): o = 0, lse = -inf
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int d0 = 64 * hw + 32 * c + 16 * hi;
          if (final_out) {
            bf16* dst = static_cast<bf16*>(a.o) + (prow + h) * kD + d0;
            reinterpret_cast<uint4*>(dst)[0] = make_uint4(0, 0, 0, 0);
            reinterpret_cast<uint4*>(dst)[1] = make_uint4(0, 0, 0, 0);
          } else {
            float4* dst = reinterpret_cast<float4*>(a.part_o + (prow + h) * kD + d0);
            for (int i = 0; i < 4; ++i) dst[i] = make_float4(0.f, 0.f, 0.f, 0.f);
          }
        }
        if (hw == 0 && hi == 0) {
          if (final_out) { if (a.lse) a.lse[prow + h] = -INFINITY; }
          else a.part_lse[prow + h] = -INFINITY;
        }
        continue;
      }
      float m_use = 0.f, l = 0.f;   // running maximum (base-2 units) and this thread's part of the row sum
      bool m_set = false;
      for (int tile = it.tile_beg; tile < it.tile_end && ok; ++tile, ++G) {
        const int sb = G % kSBuf, ms = G % kMSt;
        const bool last = tile + 1 == it.tile_end;
        ok = mbar_wait(&m_full[ms], full_par(G, kMSt), &abort_flag, lim) && ok;
        const uint4 mw = *reinterpret_cast<const uint4*>(mask[ms]);
        __syncwarp();
        if (lane == 0) mbar_arrive(&m_empty[ms]);
        ok = mbar_wait(&s_full[sb], full_par(G, kSBuf), &abort_flag, lim) && ok;
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        fence_after_sync();
        // keys 64hw + 16hi + i (x[i]) and 64hw + 32 + 16hi + i (x[16 + i]), i < 16
        uint32_t sa[16], sbv[16];
        ld16x2_x16(lane_addr + sb * kSCols + 64 * hw, sa);
        ld16x2_x16(lane_addr + sb * kSCols + 64 * hw + 32, sbv);
        tmem_wait_ld();
        fence_before_sync();   // the partner's P store into this buffer follows the exchange
        // masked keys score -inf (probability exactly 0); a tile whose keys are all
        // valid (full tiles: the common case) skips the per-key tests
        float x[32];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          x[i] = __uint_as_float(sa[i]);
          x[16 + i] = __uint_as_float(sbv[i]);
        }
        if ((mw.x & mw.y & mw.z & mw.w) != 0xffffffffu) {
          // key r's bit: word (r/2)%4, bit 2*(r/8) + r%2 (the producers' row layout)
          const uint32_t wv[4] = {mw.x, mw.y, mw.z, mw.w};
          const int sh = 16 * hw + 4 * hi;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const uint32_t wd = wv[(i >> 1) & 3];
            const int bit = 2 * (i >> 3) + (i & 1);
            x[i] = ((wd >> (sh + bit)) & 1u) ? x[i] : -INFINITY;
            x[16 + i] = ((wd >> (sh + 8 + bit)) & 1u) ? x[16 + i] : -INFINITY;
          }
        }
        float m4[4];   // four independent maximum chains
#pragma unroll
        for (int j = 0; j < 4; ++j) m4[j] = x[j];
#pragma unroll
        for (int i = 4; i < 32; ++i) m4[i & 3] = fmaxf(m4[i & 3], x[i]);
        float mt = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
        mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 16));
        mt = fmaxf(mt, exchange(mt, red[G & 1][hw][q4], red[G & 1][hw ^ 1][q4], &xbar[q4][G & 1], (G >> 1) & 1u)) * c2;
        if (!ok) break;
        fence_after_sync();
        float alpha = 1.f;
        bool resc = false;
        if (!m_set) {
          if (mt != -INFINITY) { m_use = mt; m_set = true; }   // everything so far had probability 0: O = 0
        } else if (mt > m_use + kRescaleThreshold) {
          alpha = ex2(m_use - mt);
          m_use = mt;
          resc = true;
        }
        // rescaling O waits for the O update of tile G-1.  A wait on o_bar for tile g
        // cannot alias another phase: the update of g-3 completed before S_g was
        // issued, and the update of g+3 needs P_{g+3}, which this warp writes later
        const bool wresc = __any_sync(0xffffffffu, resc);
        if (wresc) wait_o(G - 1);
        if (wresc && ok) {
          fence_after_sync();
#pragma unroll 1
          for (int c = 0; c < 2; ++c) {
            uint32_t ov[16];
            ld16x2_x16(lane_addr + kOCol + 64 * hw + 32 * c, ov);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
            st16x2_x16(lane_addr + kOCol + 64 * hw + 32 * c, ov);
          }
          tmem_wait_st();
        }
        l *= alpha;
        // probabilities as bf16 pairs: keys 64hw + [0, 32) -> P columns 32hw + [0, 16),
        // keys 64hw + 32 + [0, 32) -> 32hw + 16 + [0, 16)
        uint32_t pa[8], pb[8];
        const float mu = m_use;
        float l4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int i = 0; i < 16; i += 2) {
          const float p0 = ex2(fmaf(x[i], c2, -mu)), p1 = ex2(fmaf(x[i + 1], c2, -mu));
          const float p2 = ex2(fmaf(x[16 + i], c2, -mu)), p3 = ex2(fmaf(x[17 + i], c2, -mu));
          l4[0] += p0;
          l4[1] += p1;
          l4[2] += p2;
          l4[3] += p3;
          __nv_bfloat162 u = __floats2bfloat162_rn(p0, p1);
          __nv_bfloat162 v = __floats2bfloat162_rn(p2, p3);
          pa[i / 2] = *reinterpret_cast<uint32_t*>(&u);
          pb[i / 2] = *reinterpret_cast<uint32_t*>(&v);
        }
        l += (l4[0] + l4[1]) + (l4[2] + l4[3]);
        if (!ok) break;
        // the previous item's epilogue runs here, before this tile's P store: its last O
        // update had most of a tile's time to complete, and reading O frees the accumulator
        // before the new item's first O update can be issued
        if (pend) {
          epilogue();
          if (!ok) break;
        }
        st16x2_x8(lane_addr + sb * kSCols + 32 * hw, pa);
        st16x2_x8(lane_addr + sb * kSCols + 32 * hw + 16, pb);
        tmem_wait_st();
        fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[sb]);
        if (last) {
          pend = true;
          e_prow = prow;
          e_final = final_out;
          e_m = m_use;
          e_l = l;
          e_G = G;
        }
      }
    }
    if (pend && ok) epilogue();
  } else if (warp == kMmaWarp) {
    // ======================================================== MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(64, 128, false, false);
      constexpr uint32_t idO = idesc_bf16_f32(64, 128, false, true);
      // descriptors of the first slot of each ring; a byte offset b inside shared
      // memory (< 256 KB) adds b >> 4 to the 14-bit start-address field
      const uint64_t dq0 = desc_kmajor_sw128(smem_u32(sQ)), dk0 = desc_kmajor_sw128(smem_u32(sK));
      const uint64_t dv0 = desc_mnmajor_sw128(smem_u32(sV), kKVBytes / 2);
      // Two in-order streams scheduled by readiness: S of later tiles as K tiles and
      // S buffers free up (the O update that read a buffer's P completed), O updates
      // as probabilities arrive; neither waits for the other.
      Item s_it, p_it;
      int s_w = blockIdx.x, p_w = blockIdx.x, s_tile = 0, p_tile = 0;
      bool s_have = false, p_have = false;
      uint32_t Gs = 0, Gp = 0, nq = 0, items_done = 0;
      uint32_t idle = 0;
      unsigned long long idle_t0 = 0;
      for (;;) {
        bool prog = false;
        if (!s_have) {
          for (; s_w < n_items; s_w += gridDim.x) {
            s_it.init(a, s_w, false);
            if (s_it.n_tiles() > 0) break;
          }
          if (s_w < n_items) { s_have = true; s_tile = s_it.tile_beg; }
        }
        // ---- O stream first: O += P_G . V_G once the softmax wrote P_G (an O update frees
        // the S/P buffer that S of tile G+3 waits for)
        if (Gp < Gs) {
          if (!p_have) {
            for (; p_w < n_items; p_w += gridDim.x) {
              p_it.init(a, p_w, false);
              if (p_it.n_tiles() > 0) break;
            }
            p_have = true;
            p_tile = p_it.tile_beg;
          }
          const int pb = Gp % kSBuf, vs = Gp % kVSt;
          const bool first = p_tile == p_it.tile_beg;
          const bool c1 = !first || items_done == 0 || mbar_test_wait(&o_free, (items_done - 1) & 1u);
          const bool c2 = mbar_test_wait(&p_full[pb], full_par(Gp, kSBuf));
          const bool c3 = mbar_test_wait(&v_full[vs], full_par(Gp, kVSt));
          if (c1 & c2 & c3) {
            fence_after_sync();
            const uint64_t db = dv0 + (uint64_t)((vs * kKVBytes) >> 4);
            const uint32_t ta = tmem + pb * kSCols;
#pragma unroll
            for (int kk = 0; kk < kTile / 16; ++kk)
              mma_f16_ts(tmem + kOCol, ta + kk * 8, db + ((kk * 2048) >> 4), idO, (first && kk == 0) ? 0u : 1u);
            mma_commit(&v_empty[vs]);
            mma_commit(&o_bar[pb]);
            ++Gp;
            if (++p_tile == p_it.tile_end) {
              ++items_done;
              p_have = false;
              p_w += gridDim.x;
            }
            prog = true;
          }
        }
        // ---- S stream: S_G = Q . K_G^T into buffer G % 3 (free once the O update of G-3 completed)
        if (s_have) {
          const int sb = Gs % kSBuf, ks = Gs % kKSt, qs = nq % kQSt;
          const bool first = s_tile == s_it.tile_beg;
          // the three tests are issued together (not short-circuited), so their latencies overlap
          const bool c1 = !first || mbar_test_wait(&q_full[qs], full_par(nq, kQSt));
          const bool c2 = mbar_test_wait(&o_bar[sb], empty_par(Gs, kSBuf));
          const bool c3 = mbar_test_wait(&k_full[ks], full_par(Gs, kKSt));
          if (c1 & c2 & c3) {
            fence_after_sync();
            const uint64_t da = dq0 + (uint64_t)((qs * kQBytes) >> 4), db = dk0 + (uint64_t)((ks * kKVBytes) >> 4);
            const uint32_t d = tmem + sb * kSCols;
#pragma unroll
            for (int c = 0; c < 2; ++c)
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                mma_f16_ss(d, da + ((c * (kQBytes / 2) + kk * 32) >> 4), db + ((c * (kKVBytes / 2) + kk * 32) >> 4),
                           idS, (c | kk) != 0);
            mma_commit(&k_empty[ks]);
            mma_commit(&s_full[sb]);
            ++Gs;
            if (++s_tile == s_it.tile_end) {
              mma_commit(&q_empty[qs]);
              ++nq;
              s_have = false;
              s_w += gridDim.x;
            }
            prog = true;
          }
        }
        if (!s_have && s_w >= n_items && Gp == Gs) break;
        if (prog) {
          idle = 0;
        } else if ((++idle & 63u) == 0) {
          // nothing was ready (the issuer spins: measured faster than sleeping between
          // rounds); every 64 idle rounds, the abort flag and the time limit
          if (abort_flag) break;
          const unsigned long long now = globaltimer();
          if (idle == 64) {
            idle_t0 = now;
          } else if (now - idle_t0 > lim) {
            abort_flag = 1;
            report(HYB_ERR_TIMEOUT);
            break;
          }
        }
      }
      mma_commit(&mma_done);
      const unsigned long long t0 = globaltimer();
      while (!mbar_try_wait(&mma_done, 0) && globaltimer() - t0 < lim) {}
    }
  } else if (warp == kQWarp) {
    // ======================================================== Q tiles
    if (lane == 0) {
      prefetch_tmap(&maps.q);
      uint32_t n = 0;
      int ahead = blockIdx.x;   // next item whose Q tile is prefetched into L2
      for (int w = blockIdx.x; w < n_items; w += gridDim.x) {
        Item it;
        it.init(a, w, false);
        if (it.n_tiles() == 0) continue;
        for (; ahead < n_items && ahead <= w + 2 * (int)gridDim.x; ahead += gridDim.x) {
          const int row = ahead / a.nsplit;
          for (int c = 0; c < 2; ++c) tma_prefetch_2d(&maps.q, c * 64, row * kH);
          // the query's indexer row, read by the producers about two items from now
          if (a.idx && (a.k & 3) == 0 && (reinterpret_cast<uintptr_t>(a.idx) & 15) == 0)
            bulk_prefetch_l2(a.idx + (size_t)row * a.k, (uint32_t)a.k * 4);
        }
        const int qs = n % kQSt;
        if (!mbar_wait(&q_empty[qs], empty_par(n, kQSt), &abort_flag, lim)) break;
        mbar_expect_tx(&q_full[qs], kQBytes);
        for (int c = 0; c < 2; ++c)
          tma_load_2d(sQ + qs * kQBytes + c * (kQBytes / 2), &maps.q, &q_full[qs], c * 64, it.kl.row * kH);
        ++n;
      }
    }
  } else {
    // ======================================================== K (warps 6-9) and V (10-13) producers
    // Lane l of producer warp wi resolves the source of tile row 8*(l/2) + 2*wi + l%2;
    // the copies are coalesced: in copy i, lanes 0-15 move the 16 chunks (256 B) of
    // row 8i + 2wi and lanes 16-31 those of row 8i + 2wi + 1, each lane taking the
    // row's source index from the lane that resolved it.  The K warps' ballots of
    // valid rows form the tile's mask: word wi, bit l <-> row 8*(l/2) + 2*wi + l%2.
    const bool is_k = warp < kVWarp0;
    const int wi = warp - (is_k ? kKWarp0 : kVWarp0);
    const int r_own = 8 * (lane >> 1) + 2 * wi + (lane & 1);
    const int ch = lane & 15;   // 16-byte chunk of a 256-byte row
    const int nst = is_k ? kKSt : kVSt;
    uint64_t* fullb = is_k ? k_full : v_full;
    uint64_t* emptyb = is_k ? k_empty : v_empty;
    uint8_t* ring = is_k ? sK : sV;
    const char* csrc = static_cast<const char*>(is_k ? a.kc : a.vc);
    const char* wsrc = static_cast<const char*>(is_k ? a.kw : a.vw);
    if (wi == 0 && lane == 0) {
      prefetch_tmap(is_k ? &maps.kw : &maps.vw);
      prefetch_tmap(is_k ? &maps.kc : &maps.vc);
    }
    uint32_t G = 0;
    bool ok = true;
    for (int w = blockIdx.x; w < n_items && ok; w += gridDim.x) {
      Item it;
      it.init(a, w, false);
      const int b = div_fast(it.kl.row, a.T);
      for (int tile = it.tile_beg; tile < it.tile_end && ok; ++tile, ++G) {
        const int st = G % nst;
        const int src = key_row(a, it.kl, b, tile, r_own);   // issued before the slot wait
        const int box = tile_box_row(a, it.kl, b, tile);
        if (lane == 0) ok = mbar_wait(&emptyb[st], empty_par(G, nst), &abort_flag, lim);
        if (is_k && lane == 0 && ok) ok = mbar_wait(&m_empty[G % kMSt], empty_par(G, kMSt), &abort_flag, lim);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        uint8_t* dst = ring + st * kKVBytes;
        if (box >= 0) {
          if (wi == 0 && lane == 0) {
            const bool win = tile >= it.kl.comp_tiles;
            const CUtensorMap* map = is_k ? (win ? &maps.kw : &maps.kc) : (win ? &maps.vw : &maps.vc);
            mbar_expect_tx_only(&fullb[st], kKVBytes);
            for (int c = 0; c < 2; ++c) tma_load_2d(dst + c * (kKVBytes / 2), map, &fullb[st], c * 64, box);
          }
        } else {
          const bool win = tile >= it.kl.comp_tiles;
          const char* base = (win ? wsrc : csrc) + ch * 16;
          const int safe = win ? b * a.ring : b * a.nc_cap;   // a real row for zero-filled copies
          const uint32_t d0 = smem_u32(dst) + (ch >> 3) * (kKVBytes / 2);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int r = 8 * i + 2 * wi + (lane >> 4);
            const int sr = __shfl_sync(0xffffffffu, src, 2 * i + (lane >> 4));
            cp_async16_zfill(d0 + r * 128 + (((ch & 7) ^ (r & 7)) << 4), base + (size_t)(sr >= 0 ? sr : safe) * (kD * 2),
                             sr >= 0 ? 16u : 0u);
          }
        }
        if (!(a.test_drop_arrival && is_k && blockIdx.x == 0 && G == 0 && wi == 0 && lane == 0))
          cp_async_arrive_noinc(&fullb[st]);   // (the test hook withholds one arrival)
        if (is_k) {
          if (src == -2) report(HYB_ERR_DEVICE_CHECK);
          const uint32_t word = __ballot_sync(0xffffffffu, src >= 0 || box >= 0);
          if (lane == 0) {
            mask[G % kMSt][wi] = word;
            mbar_arrive(&m_full[G % kMSt]);
          }
        }
      }
    }
    cp_async_wait<0>();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  if (warp == kMmaWarp) tmem_dealloc(tmem, 512);
}

}  // namespace attn_hm

// Launches the heads-in-M tensor-core attention for all batch*T queries (nsplit
// slices each).  Same arguments and results as launch_attn_tc without real K/V.
inline cudaError_t launch_attn_hm(const AttnArgs& a, int batch, cudaStream_t stream) {
  using namespace attn_hm;
  Maps m;
  const uint64_t rows_q = (uint64_t)batch * a.T * kH;
  if (!make_map_bf16_2d(&m.q, a.q, rows_q, kD, kD * 2, 64, 64)) return cudaErrorInvalidValue;
  if (!make_map_bf16_2d(&m.kw, a.kw, (uint64_t)batch * a.ring, kD, kD * 2, kTile, 64)) return cudaErrorInvalidValue;
  if (!make_map_bf16_2d(&m.vw, a.vw, (uint64_t)batch * a.ring, kD, kD * 2, kTile, 64)) return cudaErrorInvalidValue;
  // Masked keys are zero-filled with an address inside their own source; with no
  // compressed cache at all the compressed source is the window ring.
  AttnArgs aa = a;
  if (a.kc == nullptr || a.vc == nullptr || a.nc_cap <= 0) {
    aa.kc = a.kw;
    aa.vc = a.vw;
    aa.nc_cap = 0;
  }
  const uint64_t rows_c = aa.nc_cap > 0 ? (uint64_t)batch * aa.nc_cap : (uint64_t)batch * a.ring;
  if (!make_map_bf16_2d(&m.kc, aa.kc, rows_c, kD, kD * 2, kTile, 64)) return cudaErrorInvalidValue;
  if (!make_map_bf16_2d(&m.vc, aa.vc, rows_c, kD, kD * 2, kTile, 64)) return cudaErrorInvalidValue;
  const int n_items = batch * a.T * a.nsplit;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = n_items < sms ? n_items : sms;
  cudaError_t e = cudaFuncSetAttribute(attn_hm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (e != cudaSuccess) return e;
  attn_hm_kernel<<<grid, kThreads, kSmem, stream>>>(m, aa, n_items);
  count_launch();
  return cudaGetLastError();
}

}  // namespace hyb
