// S3 + S4 on the 5th-generation tensor cores: shared-KV (MQA) attention of all
// 64 query heads over the selected / all compressed entries plus the sliding
// window, one joint softmax (HCA article, section "怎么压"; trdm.cn 2.1).
//
// Transposed formulation, so that every MMA has M = 128 (full rate) although
// a query has only 64 heads and, in CSA, its own key set:
//   S^T[key, h] = K_tile[key, :] . Q[h, :]        M=128 keys,  N=64 heads, K=D
//   O^T[d, h]  += V_tile^T[d, key] . P^T[key, h]  M=128 (=D),  N=64 heads, K=128 keys
// The keys of a query are processed in groups of up to 6 tiles of 128.  The
// group's S^T tiles stay in tensor memory (6 x 64 columns); the softmax warps
// (one thread per key lane) take the exact per-head maximum over the group
// (elementwise max, then a warp transpose-reduce and a 4-warp combine), rescale
// the O^T accumulator in tensor memory when a later group raises the maximum,
// then write P^T = exp2((s - m) * scale * log2 e) as a bf16 MN-major operand
// in shared memory, one 128-byte row per key.  Row sums are accumulated per
// thread and reduced across lanes once per query.
//
// Roles (192 threads, one CTA per SM, persistent over work items):
//   warp 0      producer: Q by 2-D TMA; K and V tiles by TMA gather4 (4 rows
//               per instruction, every lane issuing its own rows), compressed
//               keys and window keys in separate tiles;
//   warp 1      TMEM owner; one thread issues all MMAs and commits;
//   warps 2..5  softmax + epilogue (TMEM lane quadrant = warp % 4).
// A work item is a query or, for split-KV decode, a tile-aligned slice of its
// key list; slices write a partial (o, lse) that attn_merge combines.
#pragma once
#include "attn.cuh"
#include "common.cuh"
#include "sm100.cuh"

namespace hyb {

namespace attn_tc {

constexpr int kH = 64, kD = 128, kTile = 128;
constexpr int kGroup = 6;               // S^T tiles per group (6 x 64 TMEM columns)
constexpr int kKSt = 3, kVSt = 2, kPSt = 2;
constexpr int kThreads = 192;
constexpr int kQBytes = kH * kD * 2;                 // 16 KB (two 64-column sub-tiles)
constexpr int kKVBytes = kTile * kD * 2;             // 32 KB (two 64-column sub-tiles)
constexpr int kPBytes = kTile * kH * 2;              // 16 KB
constexpr int kSmem = kQBytes + kKSt * kKVBytes + kVSt * kKVBytes + kPSt * kPBytes + 1024;
constexpr uint32_t kOCol = kGroup * kH;              // O^T accumulator columns [384, 448)

struct Maps {
  CUtensorMap q, kc, vc, kw, vw;
};

// Per-query key list: compressed slots [0, n_comp) padded to whole tiles, then
// the window positions w0 .. w0+n_win-1.
struct KeyList {
  int row, t, vis, n_comp, n_win, w0, comp_tiles, tiles;
  __device__ void init(const AttnArgs& a, int row_) {
    row = row_;
    t = a.q_pos[row];
    vis = visible_entries(t, a.r, a.nc);
    n_comp = a.idx ? a.k : vis;
    w0 = t - a.W + 1 > 0 ? t - a.W + 1 : 0;
    n_win = a.W > 0 ? t - w0 + 1 : 0;
    comp_tiles = (n_comp + kTile - 1) / kTile;
    tiles = comp_tiles + (n_win + kTile - 1) / kTile;
  }
};

// Work item w -> (query row, tile range).
struct Item {
  KeyList kl;
  int split, tile_beg, tile_end;
  __device__ void init(const AttnArgs& a, int w) {
    const int row = w / a.nsplit;
    split = w % a.nsplit;
    kl.init(a, row);
    const int per = (kl.tiles + a.nsplit - 1) / a.nsplit;
    tile_beg = split * per;
    tile_end = min(kl.tiles, tile_beg + per);
    if (tile_beg > tile_end) tile_beg = tile_end;
  }
  __device__ int n_tiles() const { return tile_end - tile_beg; }
  __device__ int n_groups() const { return (n_tiles() + kGroup - 1) / kGroup; }
};

// Source of key v of a tile: compressed entry (is_win = false) or window slot.
// Returns -1 for padding / invalid keys (their scores are masked).
__device__ __forceinline__ int key_source(const AttnArgs& a, const KeyList& kl, int tile, int kk, bool& is_win,
                                          bool check) {
  if (tile < kl.comp_tiles) {
    is_win = false;
    const int u = tile * kTile + kk;
    if (u >= kl.n_comp) return -1;
    const int j = a.idx ? a.idx[(size_t)kl.row * a.k + u] : u;
    if (j < 0) return -1;
    if (j >= kl.vis) {
      if (check) report(HYB_ERR_DEVICE_CHECK);
      return -1;
    }
    return j;
  }
  is_win = true;
  const int u = (tile - kl.comp_tiles) * kTile + kk;
  if (u >= kl.n_win) return -1;
  return (kl.w0 + u) % a.ring;
}

__device__ __forceinline__ void named_sync_softmax() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

template <int N>
__device__ __forceinline__ void xmax_step(float* v, int lane, int mask) {
  const bool hi = (lane & mask) != 0;
#pragma unroll
  for (int i = 0; i < N / 2; ++i) {
    const float send = hi ? v[i] : v[i + N / 2];
    const float keep = hi ? v[i + N / 2] : v[i];
    v[i] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, mask));
  }
}
template <int N>
__device__ __forceinline__ void xsum_step(float* v, int lane, int mask) {
  const bool hi = (lane & mask) != 0;
#pragma unroll
  for (int i = 0; i < N / 2; ++i) {
    const float send = hi ? v[i] : v[i + N / 2];
    const float keep = hi ? v[i + N / 2] : v[i];
    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, mask);
  }
}
// After these, v[0], v[1] of lane l hold heads 2l, 2l+1 reduced over the warp.
__device__ __forceinline__ void warp_xmax64(float* v, int lane) {
  xmax_step<64>(v, lane, 16); xmax_step<32>(v, lane, 8); xmax_step<16>(v, lane, 4);
  xmax_step<8>(v, lane, 2); xmax_step<4>(v, lane, 1);
}
__device__ __forceinline__ void warp_xsum64(float* v, int lane) {
  xsum_step<64>(v, lane, 16); xsum_step<32>(v, lane, 8); xsum_step<16>(v, lane, 4);
  xsum_step<8>(v, lane, 2); xsum_step<4>(v, lane, 1);
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
      "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]),
      "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]),
      "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ Maps maps, AttnArgs a, int n_items) {
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + kQBytes;
  uint8_t* sV = sK + kKSt * kKVBytes;
  uint8_t* sP = sV + kVSt * kKVBytes;

  __shared__ uint64_t q_full, q_empty, k_full[kKSt], k_empty[kKSt], v_full[kVSt], v_empty[kVSt];
  __shared__ uint64_t s_full[kGroup], s_free, p_full[kPSt], p_empty[kPSt], o_full, o_ready, mma_done;
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;
  __shared__ float red[4][kH];
  __shared__ float m_run[kH], m_use[kH], alpha[kH], l_fin[kH];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    abort_flag = 0;
    mbar_init(&q_full, 1); mbar_init(&q_empty, 1);
    for (int s = 0; s < kKSt; ++s) { mbar_init(&k_full[s], 1); mbar_init(&k_empty[s], 1); }
    for (int s = 0; s < kVSt; ++s) { mbar_init(&v_full[s], 1); mbar_init(&v_empty[s], 1); }
    for (int s = 0; s < kGroup; ++s) mbar_init(&s_full[s], 1);
    mbar_init(&s_free, 4);
    for (int s = 0; s < kPSt; ++s) { mbar_init(&p_full[s], 4); mbar_init(&p_empty[s], 1); }
    mbar_init(&o_full, 1);
    mbar_init(&o_ready, 4);
    mbar_init(&mma_done, 1);
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(&tmem_base, 512);
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = tmem_base;
  const float c2 = a.scale * 1.4426950408889634f;  // scale * log2(e)

  if (warp == 0) {
    // ======================================================== producer
    uint32_t qn = 0, kn = 0, vn = 0;
    if (lane == 0) { prefetch_tmap(&maps.q); prefetch_tmap(&maps.kc); prefetch_tmap(&maps.kw); }
    for (int w = blockIdx.x; w < n_items && !abort_flag; w += gridDim.x) {
      Item it;
      it.init(a, w);
      if (it.n_tiles() == 0) continue;
      bool ok = true;
      if (lane == 0) {
        ok = mbar_wait(&q_empty, (qn & 1) ^ 1, &abort_flag);
        if (ok) {
          mbar_expect_tx(&q_full, kQBytes);
          for (int c = 0; c < 2; ++c) tma_load_2d(sQ + c * (kQBytes / 2), &maps.q, &q_full, c * 64, it.kl.row * kH);
        }
      }
      ++qn;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      for (int g0 = it.tile_beg; g0 < it.tile_end && ok; g0 += kGroup) {
        const int g1 = min(it.tile_end, g0 + kGroup);
        for (int pass = 0; pass < 2 && ok; ++pass) {  // K tiles of the group, then its V tiles
          for (int tile = g0; tile < g1 && ok; ++tile) {
            const int st = pass == 0 ? kn % kKSt : vn % kVSt;
            const uint32_t ph = pass == 0 ? (kn / kKSt) & 1 : (vn / kVSt) & 1;
            uint64_t* empty = pass == 0 ? &k_empty[st] : &v_empty[st];
            uint64_t* full = pass == 0 ? &k_full[st] : &v_full[st];
            uint8_t* dst = (pass == 0 ? sK : sV) + st * kKVBytes;
            if (lane == 0) {
              ok = mbar_wait(empty, ph ^ 1, &abort_flag);
              if (ok) mbar_expect_tx(full, kKVBytes);
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (ok) {
              // lane handles keys 4*lane .. 4*lane+3 of the tile
              int rows[4];
              bool win = false;
              int fallback = -1;
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                bool is_win;
                const int src = key_source(a, it.kl, tile, 4 * lane + e, is_win, pass == 0);
                win = is_win;
                rows[e] = src;
                if (src >= 0 && fallback < 0) fallback = src;
              }
              const int b = it.kl.row / a.T;
              const int base = win ? b * a.ring : b * a.nc_cap;
              if (fallback < 0) fallback = 0;
#pragma unroll
              for (int e = 0; e < 4; ++e) rows[e] = base + (rows[e] >= 0 ? rows[e] : fallback);
              const CUtensorMap* mp = pass == 0 ? (win ? &maps.kw : &maps.kc) : (win ? &maps.vw : &maps.vc);
#pragma unroll
              for (int c = 0; c < 2; ++c)
                tma_gather4(dst + c * (kKVBytes / 2) + lane * 4 * 128, mp, full, c * 64, rows[0], rows[1], rows[2],
                            rows[3]);
            }
            if (pass == 0) ++kn; else ++vn;
          }
        }
      }
    }
    // drain: loads in flight must land before the CTA can exit
    if (lane == 0 && abort_flag) {
      const unsigned long long t0 = globaltimer();
      auto drain = [&](uint64_t* bars, int nst, uint32_t n) {
        for (int s = 0; s < nst && (uint32_t)s < n; ++s) {
          const uint32_t last = s + nst * ((n - 1 - s) / nst);
          while (!mbar_try_wait(&bars[s], (last / nst) & 1) && globaltimer() - t0 < kWaitNs) {}
        }
      };
      drain(k_full, kKSt, kn);
      drain(v_full, kVSt, vn);
      if (qn > 0) while (!mbar_try_wait(&q_full, (qn - 1) & 1) && globaltimer() - t0 < kWaitNs) {}
    }
  } else if (warp == 1) {
    // ======================================================== MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc1 = idesc_bf16_f32(128, kH, false, false);
      constexpr uint32_t idesc2 = idesc_bf16_f32(128, kH, true, true);
      uint32_t qn = 0, kn = 0, vn = 0, pn = 0, gn = 0, on = 0;
      bool ok = true;
      for (int w = blockIdx.x; w < n_items && ok; w += gridDim.x) {
        Item it;
        it.init(a, w);
        if (it.n_tiles() == 0) continue;
        ok = mbar_wait(&q_full, qn & 1, &abort_flag);
        ++qn;
        bool first_pv = true;
        for (int g0 = it.tile_beg; g0 < it.tile_end && ok; g0 += kGroup) {
          const int g1 = min(it.tile_end, g0 + kGroup);
          // S^T tiles of the group (after the softmax released the previous group's)
          ok = mbar_wait(&s_free, (gn & 1) ^ 1, &abort_flag);
          for (int tile = g0; tile < g1 && ok; ++tile) {
            const int st = kn % kKSt;
            ok = mbar_wait(&k_full[st], (kn / kKSt) & 1, &abort_flag);
            if (!ok) break;
            fence_after_sync();
            const uint32_t d = tmem + (tile - g0) * kH;
            const uint32_t kbase = smem_u32(sK + st * kKVBytes);
            const uint32_t qbase = smem_u32(sQ);
#pragma unroll
            for (int c = 0; c < 2; ++c)
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                mma_f16_ss(d, desc_kmajor_sw128(kbase + c * (kKVBytes / 2) + kk * 32),
                           desc_kmajor_sw128(qbase + c * (kQBytes / 2) + kk * 32), idesc1, (c | kk) != 0);
            mma_commit(&k_empty[st]);
            ++kn;
          }
          for (int j = 0; j < kGroup; ++j) mma_commit(&s_full[j]);
          if (g1 == it.tile_end) mma_commit(&q_empty);
          ++gn;
          // O^T += V^T P^T over the group's tiles
          if (ok) ok = mbar_wait(&o_ready, on & 1, &abort_flag);
          ++on;
          for (int tile = g0; tile < g1 && ok; ++tile) {
            const int vs = vn % kVSt, ps = pn % kPSt;
            ok = mbar_wait(&v_full[vs], (vn / kVSt) & 1, &abort_flag) &&
                 mbar_wait(&p_full[ps], (pn / kPSt) & 1, &abort_flag);
            if (!ok) break;
            fence_after_sync();
            const uint32_t vbase = smem_u32(sV + vs * kKVBytes);
            const uint32_t pbase = smem_u32(sP + ps * kPBytes);
#pragma unroll
            for (int kk = 0; kk < kTile / 16; ++kk) {
              mma_f16_ss(tmem + kOCol, desc_mnmajor_sw128(vbase + kk * 2048, kKVBytes / 2),
                         desc_mnmajor_sw128(pbase + kk * 2048, 0), idesc2, (first_pv && kk == 0) ? 0u : 1u);
            }
            first_pv = false;
            mma_commit(&v_empty[vs]);
            mma_commit(&p_empty[ps]);
            ++vn;
            ++pn;
          }
          mma_commit(&o_full);
        }
      }
      mma_commit(&mma_done);
      const unsigned long long t0 = globaltimer();
      while (!mbar_try_wait(&mma_done, 0) && globaltimer() - t0 < kWaitNs) {}
    }
  } else {
    // ======================================================== softmax + epilogue
    const int quad = warp & 3;
    const int kk = quad * 32 + lane;                  // key lane within a tile / d for O^T
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const int st = tid - 64;                          // 0..127 among the softmax threads
    uint32_t gn = 0, pn = 0, on = 0;
    bool ok = true;   // on a failed wait the warps keep the same control flow (named barriers) and skip work
    for (int w = blockIdx.x; w < n_items; w += gridDim.x) {
      Item it;
      it.init(a, w);
      if (it.n_tiles() == 0) {
        // nothing visible at all (cannot happen with W >= 1): write an empty result
        if (a.nsplit == 1) {
          for (int h = 0; h < kH; ++h) store_f((bf16*)a.o + ((size_t)it.kl.row * kH + h) * kD + kk, 0.f);
          if (a.lse && st < kH) a.lse[(size_t)it.kl.row * kH + st] = -INFINITY;
        } else {
          const size_t prow = ((size_t)it.kl.row * a.nsplit + it.split) * kH;
          for (int h = 0; h < kH; ++h) a.part_o[(prow + h) * kD + kk] = 0.f;
          if (st < kH) a.part_lse[prow + st] = -INFINITY;
        }
        continue;
      }
      if (st < kH) m_run[st] = -INFINITY;
      float lp[kH];
#pragma unroll
      for (int h = 0; h < kH; ++h) lp[h] = 0.f;
      bool first_group = true;
      for (int g0 = it.tile_beg; g0 < it.tile_end; g0 += kGroup) {
        const int g1 = min(it.tile_end, g0 + kGroup);
        // ---- pass A: elementwise max over the group's tiles
        float mx[kH];
#pragma unroll
        for (int h = 0; h < kH; ++h) mx[h] = -INFINITY;
        for (int tile = g0; tile < g1; ++tile) {
          ok = mbar_wait(&s_full[tile - g0], gn & 1, &abort_flag) && ok;
          fence_after_sync();
          bool is_win;
          const bool valid = key_source(a, it.kl, tile, kk, is_win, false) >= 0;
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            uint32_t v[32];
            tmem_ld32(lane_addr + (tile - g0) * kH + c * 32, v);
            tmem_wait_ld();
            if (valid) {
#pragma unroll
              for (int e = 0; e < 32; ++e) mx[c * 32 + e] = fmaxf(mx[c * 32 + e], __uint_as_float(v[e]));
            }
          }
        }
        warp_xmax64(mx, lane);
        red[quad][2 * lane] = mx[0];
        red[quad][2 * lane + 1] = mx[1];
        named_sync_softmax();
        if (st < kH) {
          const float mg = fmaxf(fmaxf(red[0][st], red[1][st]), fmaxf(red[2][st], red[3][st]));
          const float mo = m_run[st];
          const float mn = fmaxf(mo, mg);
          alpha[st] = (mn == -INFINITY || mo == -INFINITY) ? (mo == -INFINITY ? 0.f : 1.f) : exp2f((mo - mn) * c2);
          m_run[st] = mn;
          m_use[st] = mn == -INFINITY ? 0.f : mn * c2;   // pre-multiplied by scale*log2(e)
        }
        named_sync_softmax();
        // ---- rescale the running O^T and partial sums when a later group raised the max
        if (!first_group) {
          ok = mbar_wait(&o_full, (on & 1), &abort_flag) && ok;  // previous group's PV finished
          ++on;
          fence_after_sync();
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            uint32_t v[32];
            tmem_ld32(lane_addr + kOCol + c * 32, v);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * alpha[c * 32 + e]);
            tmem_st32(lane_addr + kOCol + c * 32, v);
          }
          tmem_wait_st();
#pragma unroll
          for (int h = 0; h < kH; ++h) lp[h] *= alpha[h];
        }
        fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&o_ready);
        // ---- pass B: probabilities
        for (int tile = g0; tile < g1; ++tile) {
          bool is_win;
          const bool valid = key_source(a, it.kl, tile, kk, is_win, false) >= 0;
          const int ps = pn % kPSt;
          ok = mbar_wait(&p_empty[ps], ((pn / kPSt) & 1) ^ 1, &abort_flag) && ok;
          uint8_t* prow = sP + ps * kPBytes + kk * 128;
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            uint32_t v[32];
            tmem_ld32(lane_addr + (tile - g0) * kH + c * 32, v);
            tmem_wait_ld();
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              const float p0 = valid ? exp2f(fmaf(__uint_as_float(v[e]), c2, -m_use[c * 32 + e])) : 0.f;
              const float p1 = valid ? exp2f(fmaf(__uint_as_float(v[e + 1]), c2, -m_use[c * 32 + e + 1])) : 0.f;
              lp[c * 32 + e] += p0;
              lp[c * 32 + e + 1] += p1;
              __nv_bfloat162 b2 = __floats2bfloat162_rn(p0, p1);
              pk[e / 2] = *reinterpret_cast<uint32_t*>(&b2);
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) {  // 16-byte chunks (8 heads) 4c+q of this key's row
              const int chunk = (c * 4 + q) ^ (kk & 7);
              *reinterpret_cast<uint4*>(prow + chunk * 16) =
                  make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
            }
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&p_full[ps]);
          ++pn;
        }
        fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_free);
        ++gn;
        first_group = false;
      }
      // ---- epilogue: l = sum over lanes of lp; o = O^T / l
      warp_xsum64(lp, lane);
      red[quad][2 * lane] = lp[0];
      red[quad][2 * lane + 1] = lp[1];
      named_sync_softmax();
      if (st < kH) l_fin[st] = red[0][st] + red[1][st] + red[2][st] + red[3][st];
      named_sync_softmax();
      ok = mbar_wait(&o_full, on & 1, &abort_flag) && ok;
      ++on;
      fence_after_sync();
      const bool final_out = a.nsplit == 1;
      const size_t prow = ((size_t)it.kl.row * a.nsplit + it.split) * kH;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t v[32];
        tmem_ld32(lane_addr + kOCol + c * 32, v);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int h = c * 32 + e;
          const float l = l_fin[h];
          const float o = l > 0.f ? __uint_as_float(v[e]) / l : 0.f;
          if (final_out) store_f((bf16*)a.o + ((size_t)it.kl.row * kH + h) * kD + kk, o);
          else a.part_o[(prow + h) * kD + kk] = o;
        }
      }
      if (st < kH) {
        const float l = l_fin[st];
        const float lse = l > 0.f ? m_run[st] * a.scale + logf(l) : -INFINITY;
        if (final_out) { if (a.lse) a.lse[(size_t)it.kl.row * kH + st] = lse; }
        else a.part_lse[prow + st] = lse;
      }
      fence_before_sync();
      named_sync_softmax();   // everyone done with m_run / l_fin / O^T before the next item
    }
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

}  // namespace attn_tc

inline bool attn_tc_supported(int H, int D, const void* q, const void* kc, const void* vc, const void* kw,
                              const void* vw) {
  auto al = [](const void* p) { return p == nullptr || reinterpret_cast<uintptr_t>(p) % 16 == 0; };
  return H == attn_tc::kH && D == attn_tc::kD && al(q) && al(kc) && al(vc) && al(kw) && al(vw);
}

// Launches the tensor-core attention for all batch*T queries (nsplit slices each).
inline cudaError_t launch_attn_tc(const AttnArgs& a, int batch, cudaStream_t stream) {
  using namespace attn_tc;
  Maps m;
  const uint64_t rows_q = (uint64_t)batch * a.T * kH;
  // Padding keys gather row 0 of their source; with no compressed cache at all the
  // compressed maps point at the window ring so that row stays inside an allocation.
  const bool no_cache = a.kc == nullptr || a.vc == nullptr || a.nc_cap <= 0;
  const void* kc = no_cache ? a.kw : a.kc;
  const void* vc = no_cache ? a.vw : a.vc;
  const uint64_t rows_c = no_cache ? (uint64_t)batch * a.ring : (uint64_t)batch * a.nc_cap;
  if (!make_map_bf16_2d(&m.q, a.q, rows_q, kD, kD * 2, 64, 64)) return cudaErrorInvalidValue;
  if (!make_map_bf16_2d(&m.kc, kc, rows_c, kD, kD * 2, 1, 64)) return cudaErrorInvalidValue;
  if (!make_map_bf16_2d(&m.vc, vc, rows_c, kD, kD * 2, 1, 64)) return cudaErrorInvalidValue;
  if (!make_map_bf16_2d(&m.kw, a.kw, (uint64_t)batch * a.ring, kD, kD * 2, 1, 64)) return cudaErrorInvalidValue;
  if (!make_map_bf16_2d(&m.vw, a.vw, (uint64_t)batch * a.ring, kD, kD * 2, 1, 64)) return cudaErrorInvalidValue;
  const int n_items = batch * a.T * a.nsplit;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = n_items < sms ? n_items : sms;
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (e != cudaSuccess) return e;
  attn_tc_kernel<<<grid, kThreads, kSmem, stream>>>(m, a, n_items);
  count_launch();
  return cudaGetLastError();
}

}  // namespace hyb
