// S3 + S4 on the 5th-generation tensor cores: shared-KV (MQA) attention of all
// 64 query heads over the selected / all compressed entries plus the sliding
// window, one joint softmax (HCA article, section "怎么压"; trdm.cn 2.1).
//
// Transposed formulation, so that every MMA has M = 128 (full rate) although a
// query has only 64 heads and, in CSA, its own key set:
//   S^T[key, h] = K_tile[key, :] . Q[h, :]        M=128 keys, N=64 heads, K=D
//   O^T[d, h]  += V_tile^T[d, key] . P^T[key, h]  M=128 (=D), N=64 heads, K=128 keys
// A query's keys (compressed entries first, then window positions, each padded
// to whole tiles of 128) are processed in groups of up to 3 tiles.
//
// Roles (16 warps, one CTA per SM, persistent over work items):
//   warp 1      key tables: turns each group's key list (indexer output or the
//               dense range, then the window) into source rows in shared memory
//               one group ahead, so no role waits on a global index load; also
//               loads each query's Q tile (2-D TMA, double-buffered);
//   warps 2-6   K tiles, warps 7-11 V tiles: gathered rows are copied with
//               16-byte cp.async by all 96 lanes (the per-SM gather rate grows
//               with the number of issuing warps), written in the 128-byte
//               swizzled layout; a window tile whose rows are consecutive is one
//               2-D TMA box per 64-column half instead.  Every producer lane
//               makes one asynchronous arrival per tile that the hardware
//               performs when the lane's copies have landed;
//   warp 0      TMEM owner; one thread issues every MMA: S^T of group g+1 is
//               issued before O^T of group g, so the tensor core computes the
//               next group's scores while the softmax warps turn the current
//               scores into probabilities;
//   warps 12-19 softmax and epilogue: thread = key lane (TMEM lane quadrant =
//               warp % 4), warps 12-15 own heads 0-31 and warps 16-19 heads 32-63.
// Tensor memory: two S^T buffers (3 tiles x 64 columns) and two O^T
// accumulators (64 columns), 512 columns in all.
//
// Softmax: per group, the per-head maximum over the group's keys (elementwise
// max over the tiles, a warp transpose-reduce across key lanes, a 4-warp
// combine).  The running maximum only moves when a group exceeds it by more
// than 8 (base-2 exponent units), in which case O^T and the per-thread row sums
// are rescaled; otherwise probabilities are taken against the stale maximum
// (they stay below 2^8).  P^T is written as a bf16 MN-major operand in shared
// memory, one 128-byte row per key.  Row sums are reduced across key lanes once
// per query.  The normalised bf16 output tile o[h][d] is staged in shared memory
// and written to global memory by one bulk copy on the TMA engine; keys masked
// out (indexer padding) are zero-filled by the producers without a global read.  A work item is a query or, for split-KV decode, a tile-aligned
// slice of its keys; slices write partial (o, lse) pairs that attn_merge combines.
#pragma once
#include "attn.cuh"
#include "common.cuh"
#include "sm100.cuh"

namespace hyb {

namespace attn_tc {

constexpr int kH = 64, kD = 128, kTile = 128;
constexpr int kGT = 3;                                  // tiles per group
// One Q slot (the next query's Q loads while the softmax finishes the current
// one), three V slots (a V tile may load while the O^T update two tiles back
// still waits for probabilities), four key-table slots.
constexpr int kQSt = 1, kKSt = 2, kVSt = 3, kPSt = 2, kTbl = 4;
constexpr int kProdWarps = 3;                           // per tensor (K, V)
constexpr int kProdLanes = kProdWarps * 32;
constexpr int kSmxWarp0 = (2 + 2 * kProdWarps + 3) / 4 * 4;   // first softmax warp (warpgroup-aligned)
constexpr int kThreads = (kSmxWarp0 + 8) * 32;
// Register split per warpgroup (setmaxnreg): warps below kSmxWarp0 drop to kRegLow,
// the 8 softmax warps rise to kRegHigh; the sum stays within the launch allocation
// (65536 / kThreads rounded down to a multiple of 8, per thread).
constexpr int kRegLow = 56, kRegHigh = 200;
static_assert(kRegLow * 32 * kSmxWarp0 + kRegHigh * 256 <= (65536 / kThreads) / 8 * 8 * kThreads,
              "register split exceeds the launch allocation");
constexpr int kQBytes = kH * kD * 2;                    // 16 KB, two 64-column sub-tiles
constexpr int kKVBytes = kTile * kD * 2;                // 32 KB, two 64-column sub-tiles
constexpr int kPBytes = kTile * kH * 2;                 // 16 KB
constexpr int kOBytes = kH * kD * 2;                    // 16 KB bf16 output tile [h][d], staged in P slot 0
static_assert(kOBytes <= kPBytes, "the output tile is staged in a P slot");
constexpr int kSmem = kQSt * kQBytes + kKSt * kKVBytes + kVSt * kKVBytes + kPSt * kPBytes + 1024;
constexpr uint32_t kSCols = kGT * kH;                   // 192 columns per S^T buffer
constexpr uint32_t kOCol = 2 * kSCols;                  // O^T buffers at 384 and 448
constexpr float kRescaleThreshold = 8.f;                // base-2 units
constexpr int kTblArrivals = 2 * kProdLanes + 256;      // K producers, V producers, softmax lanes

struct Maps {
  CUtensorMap q;        // [batch*T*H, D], 64 x 64 boxes
  CUtensorMap kw, vw;   // [batch*ring, D], 128-row x 64-column boxes (contiguous window tiles)
  CUtensorMap kc, vc;   // [batch*nc_cap, D], same boxes (full tiles of a dense compressed range)
};

// Per-query key list: compressed slots [0, n_comp) padded to whole tiles, then
// the window positions w0 .. w0+n_win-1.
// x / d and x % d for d > 0, with the common power-of-two divisors (r = 4 or 128,
// ring lengths, one split) taking a shift instead of a division: every warp of the
// attention kernels computes this per work item.
__device__ __forceinline__ int div_fast(int x, int d) { return (d & (d - 1)) == 0 ? x >> (__ffs(d) - 1) : x / d; }
__device__ __forceinline__ int mod_fast(int x, int d) { return (d & (d - 1)) == 0 ? x & (d - 1) : x % d; }

struct KeyList {
  int row, t, vis, n_comp, n_win, w0, w0_slot, comp_tiles, tiles;   // w0_slot = w0 mod ring
  __device__ void init(const AttnArgs& a, int row_, bool real_kv) {
    row = row_;
    t = a.q_pos[row];
    const int v = div_fast(t + 1, a.r);
    vis = v < a.nc ? v : a.nc;
    n_comp = a.idx ? (real_kv ? a.k * a.r : a.k) : vis;
    w0 = t - a.W + 1 > 0 ? t - a.W + 1 : 0;
    w0_slot = mod_fast(w0, a.ring);
    n_win = a.W > 0 ? t - w0 + 1 : 0;
    comp_tiles = (n_comp + kTile - 1) / kTile;
    tiles = comp_tiles + (n_win + kTile - 1) / kTile;
  }
};

// Work item w -> (query row, tile range).
struct Item {
  KeyList kl;
  int split, tile_beg, tile_end;
  __device__ void init(const AttnArgs& a, int w, bool real_kv) {
    const int row = a.nsplit == 1 ? w : w / a.nsplit;
    split = a.nsplit == 1 ? 0 : w - row * a.nsplit;
    kl.init(a, row, real_kv);
    const int per = a.nsplit == 1 ? kl.tiles : (kl.tiles + a.nsplit - 1) / a.nsplit;
    tile_beg = split * per;
    tile_end = min(kl.tiles, tile_beg + per);
    if (tile_beg > tile_end) tile_beg = tile_end;
  }
  __device__ int n_tiles() const { return tile_end - tile_beg; }
};

// Indexer entry behind key kk of compressed tile `tile` (the dense range when
// there is no indexer; with real K/V, key u is token u mod r of entry u / r);
// -1 for window tiles and padding.  A pure load, so a group's loads can all be
// in flight together.
__device__ __forceinline__ int key_entry(const AttnArgs& a, const KeyList& kl, int tile, int kk, bool real_kv) {
  const int u = tile * kTile + kk;
  if (tile >= kl.comp_tiles || u >= kl.n_comp) return -1;
  if (!a.idx) return u;
  return __ldg(a.idx + (size_t)kl.row * a.k + (real_kv ? u / a.r : u));
}

// Source of key kk of a tile: entry index (compressed, from its entry e) or ring
// slot (window); -1 for padding / masked keys, -2 for an entry outside the
// visible range.
__device__ __forceinline__ int key_source(const AttnArgs& a, const KeyList& kl, int tile, int kk, int e,
                                          bool real_kv) {
  if (tile < kl.comp_tiles) {
    if (e < 0) return -1;
    if (e >= kl.vis) return -2;
    if (!real_kv) return e;
    const int tok = e * a.r + (tile * kTile + kk) % a.r;   // a raw token of the entry (<= t)
    if (tok >= kl.w0) return -1;                            // the window holds it already
    if (tok <= kl.t - a.ring) return -2;                    // no longer in the ring
    return tok % a.ring;
  }
  const int u = (tile - kl.comp_tiles) * kTile + kk;
  if (u >= kl.n_win) return -1;
  return (kl.w0 + u) % a.ring;
}

struct KeyTable {
  int rows[kTbl][kGT * kTile];   // source row, -1 = masked key
  int safe[kTbl][kGT];           // a real row of the tile's source for masked keys
  int win[kTbl][kGT];            // 1 if the tile holds window keys
  int first[kTbl][kGT];          // >= 0: the tile is rows first .. first+127 of the window source
};

__device__ __forceinline__ void named_sync_softmax() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

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
// 32 values per lane -> v[0] of lane l holds element l reduced over the warp.
__device__ __forceinline__ void warp_xmax32(float* v, int lane) {
  xmax_step<32>(v, lane, 16); xmax_step<16>(v, lane, 8); xmax_step<8>(v, lane, 4);
  xmax_step<4>(v, lane, 2); xmax_step<2>(v, lane, 1);
}
__device__ __forceinline__ void warp_xsum32(float* v, int lane) {
  xsum_step<32>(v, lane, 16); xsum_step<16>(v, lane, 8); xsum_step<8>(v, lane, 4);
  xsum_step<4>(v, lane, 2); xsum_step<2>(v, lane, 1);
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
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2-slot ring helpers: use u of a slot -> phase parity.
__device__ __forceinline__ uint32_t full_par(uint32_t n, int nst) { return (n / nst) & 1u; }
__device__ __forceinline__ uint32_t empty_par(uint32_t n, int nst) { return ((n / nst) & 1u) ^ 1u; }

struct PendingPV {
  int valid, ob, ntiles, first, x;   // x: parity of the group's index within its query (o_full barrier)
};

template <bool RKV>   // the real-K/V reading (a compile-time switch: no cost to the other path)
__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ Maps maps, AttnArgs a, int n_items) {
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + kQSt * kQBytes;
  uint8_t* sV = sK + kKSt * kKVBytes;
  uint8_t* sP = sV + kVSt * kKVBytes;
  uint8_t* sO = sP;   // output staging: P slot 0, idle once the query's last O^T update is done

  __shared__ uint64_t q_full[kQSt], q_empty[kQSt], k_full[kKSt], k_empty[kKSt], v_full[kVSt], v_empty[kVSt];
  // o_full[ob][x]: O^T update of a group of the query in accumulator ob complete, x = parity of
  // the group's index; two barriers let the softmax lag one group behind without phase aliasing
  __shared__ uint64_t s_full[2], s_free[2], p_full[kPSt], p_empty[kPSt], o_full[2][2], o_ready[2];
  __shared__ uint64_t t_full[kTbl], t_empty[kTbl], mma_done;
  __shared__ KeyTable tbl;
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;
  __shared__ float red[2][4][32];
  __shared__ float m_run[kH], alpha_s[kH];
  __shared__ __align__(16) float m_use[kH];
  __shared__ __align__(16) float l_inv[kH];   // 1 / row sum, 0 for a head with no key
  __shared__ int resc_flag[2];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    abort_flag = 0;
    for (int s = 0; s < kQSt; ++s) { mbar_init(&q_full[s], 1); mbar_init(&q_empty[s], 1); }
    for (int s = 0; s < kKSt; ++s) { mbar_init(&k_full[s], kProdLanes); mbar_init(&k_empty[s], 1); }
    for (int s = 0; s < kVSt; ++s) { mbar_init(&v_full[s], kProdLanes); mbar_init(&v_empty[s], 1); }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1); mbar_init(&s_free[s], 8);
      mbar_init(&o_full[s][0], 1); mbar_init(&o_full[s][1], 1); mbar_init(&o_ready[s], 8);
    }
    for (int s = 0; s < kPSt; ++s) { mbar_init(&p_full[s], 8); mbar_init(&p_empty[s], 1); }
    for (int s = 0; s < kTbl; ++s) { mbar_init(&t_full[s], 32); mbar_init(&t_empty[s], kTblArrivals); }
    mbar_init(&mma_done, 1);
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(&tmem_base, 512);
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = tmem_base;
  const float c2 = a.scale * 1.4426950408889634f;  // scale * log2(e)

  // Register split per warpgroup (kRegLow / kRegHigh, see their definition).
  if (warp < kSmxWarp0) {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegLow) : "memory");
  if (warp == 1) {
    // ======================================================== key tables and Q
    // Q tiles are queued and issued by lane 0 whenever their slot is free, so
    // building tables never waits for a Q slot.
    constexpr int kQQ = 16;                 // queued Q loads (>= items a full table ring can span)
    int qrow[kQQ];
    uint32_t G = 0, n = 0, q_next = 0;
    auto service_q = [&]() {
      if (lane != 0) return;
      while (q_next < n && mbar_test_wait(&q_empty[q_next % kQSt], empty_par(q_next, kQSt))) {
        const int qb = q_next % kQSt;
        mbar_expect_tx(&q_full[qb], kQBytes);
        for (int c = 0; c < 2; ++c)
          tma_load_2d(sQ + qb * kQBytes + c * (kQBytes / 2), &maps.q, &q_full[qb], c * 64, qrow[q_next % kQQ] * kH);
        ++q_next;
      }
    };
    // Polls `bar` while serving the Q queue (a non-suspending test, so that a Q slot
    // freed meanwhile is refilled at once); false on abort or time-out.
    auto wait_serving = [&](uint64_t* bar, uint32_t par) {
      const unsigned long long t0 = globaltimer();
      for (uint32_t it = 0;; ++it) {
        service_q();
        if (mbar_test_wait(bar, par)) return true;
        if ((it & 63u) == 63u) {
          if (abort_flag) return false;
          if (globaltimer() - t0 > kWaitNs) {
            abort_flag = 1;
            report(HYB_ERR_TIMEOUT);
            return false;
          }
        }
      }
    };
    for (int w = blockIdx.x; w < n_items && !abort_flag; w += gridDim.x) {
      Item it;
      it.init(a, w, RKV);
      if (it.n_tiles() == 0) continue;
      const int b = it.kl.row / a.T;
      if (lane == 0) {   // (q_next is lane 0's; the queue cannot fill while the table ring holds fewer groups)
        if (n - q_next >= kQQ && wait_serving(&q_empty[q_next % kQSt], empty_par(q_next, kQSt))) service_q();
        qrow[n % kQQ] = it.kl.row;
        for (int c = 0; c < 2; ++c) tma_prefetch_2d(&maps.q, c * 64, it.kl.row * kH);   // into L2, ahead of its slot
      }
      ++n;
      service_q();
      for (int g0 = it.tile_beg; g0 < it.tile_end; g0 += kGT, ++G) {
        const int nt = min(kGT, it.tile_end - g0);
        const int slot = G % kTbl;
        // the group's indexer loads are issued before the wait for its table slot
        int src[kGT][4];
#pragma unroll
        for (int j = 0; j < kGT; ++j)
#pragma unroll
          for (int i = 0; i < 4; ++i) src[j][i] = j < nt ? key_entry(a, it.kl, g0 + j, lane + 32 * i, RKV) : -1;
        if (!wait_serving(&t_empty[slot], empty_par(G, kTbl))) break;
        bool bad = false;
#pragma unroll
        for (int j = 0; j < kGT; ++j)
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int sj = j < nt ? key_source(a, it.kl, g0 + j, lane + 32 * i, src[j][i], RKV) : -1;
            bad |= sj == -2;
            src[j][i] = sj < 0 ? -1 : sj;
          }
        if (bad) report(HYB_ERR_DEVICE_CHECK);
#pragma unroll
        for (int j = 0; j < kGT; ++j) {
          if (j >= nt) break;
          const bool win = g0 + j >= it.kl.comp_tiles;
          const bool from_ring = win || RKV;   // real K/V: compressed keys are raw tokens of the ring
          const int base = from_ring ? b * a.ring : b * a.nc_cap;
#pragma unroll
          for (int i = 0; i < 4; ++i) tbl.rows[slot][j * kTile + lane + 32 * i] = src[j][i] >= 0 ? base + src[j][i] : -1;
          if (lane == 0) {
            tbl.safe[slot][j] = base;
            tbl.win[slot][j] = from_ring ? 1 : 0;
            int first = -1;
            if (win) {   // window positions are consecutive rows unless the ring wraps inside the tile
              const int s0 = (it.kl.w0 + (g0 + j - it.kl.comp_tiles) * kTile) % a.ring;
              if (s0 + kTile <= a.ring) first = base + s0;
            } else if (!a.idx && (g0 + j + 1) * kTile <= it.kl.n_comp) {
              first = base + (g0 + j) * kTile;   // a full tile of the dense compressed range
            }
            tbl.first[slot][j] = first;
          }
        }
        mbar_arrive(&t_full[slot]);
      }
    }
    if (lane == 0) {   // issue the Q tiles still queued
      const unsigned long long t0 = globaltimer();
      while (q_next < n && !abort_flag) {
        service_q();
        if (globaltimer() - t0 > kWaitNs) {
          abort_flag = 1;
          report(HYB_ERR_TIMEOUT);
        }
      }
    }
  } else if (warp >= 2) {
    // ======================================================== K and V producers (kProdWarps each)
    const bool is_k = warp < 2 + kProdWarps;
    const int plane = (warp - (is_k ? 2 : 2 + kProdWarps)) * 32 + lane;   // 0 .. kProdLanes-1
    uint32_t G = 0, tiles = 0;
    bool ok = true;
    if (plane == 0) {
      prefetch_tmap(is_k ? &maps.kw : &maps.vw);
      prefetch_tmap(is_k ? &maps.kc : &maps.vc);
    }
    for (int w = blockIdx.x; w < n_items && ok; w += gridDim.x) {
      Item it;
      it.init(a, w, RKV);
      if (it.n_tiles() == 0) continue;
      for (int g0 = it.tile_beg; g0 < it.tile_end && ok; g0 += kGT, ++G) {
        const int nt = min(kGT, it.tile_end - g0);
        const int slot = G % kTbl;
        ok = mbar_wait(&t_full[slot], full_par(G, kTbl), &abort_flag);
        for (int j = 0; j < nt && ok; ++j, ++tiles) {
          const int nst = is_k ? kKSt : kVSt;
          const int st = tiles % nst;
          uint64_t* empty = is_k ? &k_empty[st] : &v_empty[st];
          uint64_t* full = is_k ? &k_full[st] : &v_full[st];
          uint8_t* dst = (is_k ? sK : sV) + st * kKVBytes;
          if (lane == 0) ok = mbar_wait(empty, empty_par(tiles, nst), &abort_flag);
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) break;
          const int first = tbl.first[slot][j];
          if (first >= 0) {
            // consecutive rows (window, or dense compressed entries): one 2-D TMA box per 64-column half
            if (plane == 0) {
              const bool win = tbl.win[slot][j] != 0;
              const CUtensorMap* map = is_k ? (win ? &maps.kw : &maps.kc) : (win ? &maps.vw : &maps.vc);
              mbar_expect_tx_only(full, kKVBytes);
              for (int c = 0; c < 2; ++c) tma_load_2d(dst + c * (kKVBytes / 2), map, full, c * 64, first);
            }
          } else {
            // gathered rows: a lane owns one 16-byte chunk position of a row in both
            // 64-column halves; all of its row indices are read from the table first
            // so that its copies issue back to back (a shared-memory read between
            // copies halves the gather rate).  Copies are written with the 128-byte
            // swizzle the MMA descriptors expect; a masked key's row is zero-filled
            // without reading global memory.
            constexpr int kTasks = kTile * 8;                       // (row, chunk) pairs per tile
            constexpr int kIt = (kTasks + kProdLanes - 1) / kProdLanes;
            const int safe = tbl.safe[slot][j];
            const bool win = tbl.win[slot][j] != 0;
            const char* src = static_cast<const char*>(is_k ? (win ? a.kw : a.kc) : (win ? a.vw : a.vc));
            const int* trow = tbl.rows[slot] + j * kTile;
            const uint32_t dbase = smem_u32(dst);
            int rw[kIt];
#pragma unroll
            for (int i = 0; i < kIt; ++i) {
              const int q = i * kProdLanes + plane;
              rw[i] = q < kTasks ? trow[q >> 3] : -1;
            }
#pragma unroll
            for (int i = 0; i < kIt; ++i) {
              const int q = i * kProdLanes + plane;
              if (q < kTasks) {
                const int r = q >> 3, ch = q & 7;
                const char* row = src + (size_t)(rw[i] >= 0 ? rw[i] : safe) * (kD * 2) + ch * 16;
                const uint32_t d = dbase + r * 128 + ((ch ^ (r & 7)) << 4);
                const uint32_t nb = rw[i] >= 0 ? 16u : 0u;
                cp_async16_zfill(d, row, nb);
                cp_async16_zfill(d + kKVBytes / 2, row + 128, nb);
              }
            }
          }
          cp_async_arrive_noinc(full);   // arrives when this lane's copies of the tile have landed
        }
        mbar_arrive(&t_empty[slot]);
      }
    }
    cp_async_wait<0>();
  } else {
    // ======================================================== MMA issuer
    // Two in-order streams, scheduled by readiness instead of program order: the
    // S^T tiles of the groups (K tiles as they land) and the O^T += V^T P^T tiles
    // of groups whose probabilities are being produced.  Neither waits for the
    // other, so the last O^T update of a query does not wait for the next
    // query's K tiles, and S^T of the next group overlaps the current softmax.
    if (lane == 0) {
      constexpr uint32_t idesc1 = idesc_bf16_f32(128, kH, false, false);
      constexpr uint32_t idesc2 = idesc_bf16_f32(128, kH, true, true);
      constexpr int kRing = 4;
      // S stream
      Item s_it;
      int s_w = blockIdx.x, s_g0 = 0, s_nt = 0, s_j = 0, s_gi = 0;
      bool s_have = false, s_first = true, s_open = false;
      uint32_t Gs = 0, ns = 0, kt = 0;
      // PV stream: groups whose S^T has been issued, oldest first
      PendingPV ring[kRing];
      int ph = 0, pc = 0, p_j = 0;
      bool p_open = false;
      uint32_t vt = 0, pt = 0, pg = 0;   // pg: groups whose O^T update was opened
      uint32_t idle = 0;
      unsigned long long idle_t0 = 0;
      for (;;) {
        bool prog = false;
        if (!s_have) {
          for (; s_w < n_items; s_w += gridDim.x) {
            s_it.init(a, s_w, RKV);
            if (s_it.n_tiles() > 0) break;
          }
          if (s_w < n_items) {
            s_have = true;
            s_first = true;
            s_gi = 0;
            s_open = false;
            s_g0 = s_it.tile_beg;
          }
        }
        if (s_have && pc < kRing) {
          const int sb = Gs % 2, qb = ns % kQSt;
          if (!s_open && mbar_test_wait(&s_free[sb], empty_par(Gs, 2)) &&
              (!s_first || mbar_test_wait(&q_full[qb], full_par(ns, kQSt)))) {
            s_open = true;
            s_nt = min(kGT, s_it.tile_end - s_g0);
            s_j = 0;
          }
          if (s_open) {
            while (s_j < s_nt) {
              const int ks = kt % kKSt;
              if (!mbar_test_wait(&k_full[ks], full_par(kt, kKSt))) break;
              fence_after_sync();
              fence_async_shared();
              const uint32_t d = tmem + sb * kSCols + s_j * kH;
              const uint32_t kbase = smem_u32(sK + ks * kKVBytes);
              const uint32_t qbase = smem_u32(sQ + qb * kQBytes);
#pragma unroll
              for (int c = 0; c < 2; ++c)
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                  mma_f16_ss(d, desc_kmajor_sw128(kbase + c * (kKVBytes / 2) + kk * 32),
                             desc_kmajor_sw128(qbase + c * (kQBytes / 2) + kk * 32), idesc1, (c | kk) != 0);
              mma_commit(&k_empty[ks]);
              ++kt;
              ++s_j;
              prog = true;
            }
            if (s_j == s_nt) {
              const bool last = s_g0 + kGT >= s_it.tile_end;
              mma_commit(&s_full[sb]);
              if (last) mma_commit(&q_empty[qb]);
              ring[(ph + pc) % kRing] = PendingPV{1, static_cast<int>(ns % 2), s_nt, s_first ? 1 : 0, s_gi & 1};
              ++s_gi;
              ++pc;
              ++Gs;
              s_first = false;
              s_open = false;
              s_g0 += kGT;
              if (last) {
                s_have = false;
                ++ns;
                s_w += gridDim.x;
              }
              prog = true;
            }
          }
        }
        if (pc > 0) {
          const PendingPV pv = ring[ph];
          if (!p_open && mbar_test_wait(&o_ready[pg & 1], full_par(pg, 2))) {
            ++pg;
            p_open = true;
            p_j = 0;
            prog = true;
          }
          if (p_open) {
            while (p_j < pv.ntiles) {
              const int vs = vt % kVSt, ps = pt % kPSt;
              if (!mbar_test_wait(&v_full[vs], full_par(vt, kVSt)) || !mbar_test_wait(&p_full[ps], full_par(pt, kPSt))) break;
              fence_after_sync();
              fence_async_shared();
              const uint32_t vbase = smem_u32(sV + vs * kKVBytes);
              const uint32_t pbase = smem_u32(sP + ps * kPBytes);
#pragma unroll
              for (int kk = 0; kk < kTile / 16; ++kk)
                mma_f16_ss(tmem + kOCol + pv.ob * kH, desc_mnmajor_sw128(vbase + kk * 2048, kKVBytes / 2),
                           desc_mnmajor_sw128(pbase + kk * 2048, 0), idesc2, (pv.first && p_j == 0 && kk == 0) ? 0u : 1u);
              mma_commit(&v_empty[vs]);
              mma_commit(&p_empty[ps]);
              ++vt;
              ++pt;
              ++p_j;
              prog = true;
            }
            if (p_j == pv.ntiles) {
              mma_commit(&o_full[pv.ob][pv.x]);
              p_open = false;
              ph = (ph + 1) % kRing;
              --pc;
              prog = true;
            }
          }
        }
        if (!s_have && s_w >= n_items && pc == 0) break;
        if (prog) {
          idle = 0;
        } else if ((++idle & 63u) == 0) {   // no progress: check the abort flag and the time limit
          if (abort_flag) break;
          const unsigned long long now = globaltimer();
          if (idle == 64) {
            idle_t0 = now;
          } else if (now - idle_t0 > kWaitNs) {
            abort_flag = 1;
            report(HYB_ERR_TIMEOUT);
            break;
          }
        }
      }
      mma_commit(&mma_done);
      const unsigned long long t0 = globaltimer();
      while (!mbar_try_wait(&mma_done, 0) && globaltimer() - t0 < kWaitNs) {}
    }
  }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegHigh) : "memory");
    // ======================================================== softmax + epilogue (8 warps from kSmxWarp0)
    const int quad = warp & 3;
    const int hf = (warp - kSmxWarp0) >> 2;           // head half: heads 32*hf .. 32*hf+31
    const int kk = quad * 32 + lane;                  // key lane of a tile; head-dim lane of O^T
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    uint32_t G = 0, n = 0, pt = 0;
    uint32_t ofw[2][2] = {{0, 0}, {0, 0}};   // phases of o_full[ob][x] consumed
    bool ok = true;   // on a failed wait the warps keep the same control flow (named barriers) and skip work
    for (int w = blockIdx.x; w < n_items; w += gridDim.x) {
      Item it;
      it.init(a, w, RKV);
      const bool final_out = a.nsplit == 1;
      const size_t prow = final_out ? (size_t)it.kl.row * kH : ((size_t)it.kl.row * a.nsplit + it.split) * kH;
      if (it.n_tiles() == 0) {
        // no key at all (impossible with W >= 1 in prefill; empty slices in split-KV)
#pragma unroll 4
        for (int e = 0; e < 32; ++e) {
          const int h = hf * 32 + e;
          if (final_out) store_f((bf16*)a.o + (prow + h) * kD + kk, 0.f);
          else a.part_o[(prow + h) * kD + kk] = 0.f;
        }
        if (quad == 0) {
          const int h = hf * 32 + lane;
          if (final_out) { if (a.lse) a.lse[prow + h] = -INFINITY; }
          else a.part_lse[prow + h] = -INFINITY;
        }
        continue;
      }
      const int ob = n % 2;
      float lp[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) lp[e] = 0.f;
      bool first = true;
      int gi = 0, cons = 0;   // group index within the query; O^T updates consumed so far
      for (int g0 = it.tile_beg; g0 < it.tile_end; g0 += kGT, ++G) {
        const int nt = min(kGT, it.tile_end - g0);
        const bool last = g0 + kGT >= it.tile_end;
        const int sb = G % 2, slot = G % kTbl;
        ok = mbar_wait(&t_full[slot], full_par(G, kTbl), &abort_flag) && ok;
        uint32_t vmask = 0;   // bit j: this thread's key of tile j is a real key
#pragma unroll
        for (int j = 0; j < kGT; ++j) vmask |= (j < nt && tbl.rows[slot][j * kTile + kk] >= 0) ? (1u << j) : 0u;
        mbar_arrive(&t_empty[slot]);
        ok = mbar_wait(&s_full[sb], full_par(G, 2), &abort_flag) && ok;
        fence_after_sync();
        // ---- pass A: elementwise max over the group's tiles, then across key lanes
        float mx[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) mx[e] = -INFINITY;
#pragma unroll 1
        for (int j = 0; j < nt; ++j) {
          uint32_t v[32];
          tmem_ld32(lane_addr + sb * kSCols + j * kH + hf * 32, v);
          tmem_wait_ld();
          if (vmask & (1u << j)) {
#pragma unroll
            for (int e = 0; e < 32; ++e) mx[e] = fmaxf(mx[e], __uint_as_float(v[e]));
          }
        }
        warp_xmax32(mx, lane);
        red[hf][quad][lane] = mx[0] * c2;
        // P slot 0 held the previous query's output tile: its bulk store must have
        // read it before this query's probabilities are written there
        if (first && warp == kSmxWarp0 && lane == 0) bulk_wait_read_all();
        named_sync_softmax();
        if (quad == 0) {
          const int h = hf * 32 + lane;
          const float g = fmaxf(fmaxf(red[hf][0][lane], red[hf][1][lane]), fmaxf(red[hf][2][lane], red[hf][3][lane]));
          const float mo = m_run[h];
          float mn = mo, al = 1.f;
          bool resc = false;
          if (first) {
            mn = g;
          } else if (g > mo + kRescaleThreshold || (mo == -INFINITY && g != -INFINITY)) {
            mn = g;
            al = mo == -INFINITY ? 0.f : ex2_approx(mo - mn);
            resc = true;
          }
          m_run[h] = mn;
          m_use[h] = mn == -INFINITY ? 0.f : mn;
          alpha_s[h] = al;
          const unsigned any = __ballot_sync(0xffffffffu, resc);
          if (lane == 0) resc_flag[hf] = any != 0;
        }
        named_sync_softmax();
        // ---- O^T updates this group needs complete: two groups back (so that no o_full
        // barrier runs two phases ahead of this thread), one back when O^T is rescaled
        {
          const int need = resc_flag[hf] ? gi - 1 : gi - 2;
          while (cons <= need) {
            ok = mbar_wait(&o_full[ob][cons & 1], ofw[ob][cons & 1] & 1u, &abort_flag) && ok;
            ++ofw[ob][cons & 1];
            ++cons;
          }
        }
        if (!first) {
          fence_after_sync();
          if (resc_flag[hf]) {
            uint32_t v[32];
            const uint32_t oaddr = lane_addr + kOCol + ob * kH + hf * 32;
            tmem_ld32(oaddr, v);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const float al = alpha_s[hf * 32 + e];
              v[e] = __float_as_uint(__uint_as_float(v[e]) * al);
              lp[e] *= al;
            }
            tmem_st32(oaddr, v);
            tmem_wait_st();
          }
        }
        fence_before_sync();
        __syncwarp();
        // by the parity of the group's global index: the arrival for group G + 2 needs the O^T
        // update of group G (the wait above, or the previous query's epilogue), so the issuer
        // has consumed this barrier's previous phase before the next one completes
        if (lane == 0) mbar_arrive(&o_ready[G & 1]);
        // ---- pass B: probabilities into P^T
        const float* mu = m_use + hf * 32;
#pragma unroll 1
        for (int j = 0; j < nt; ++j) {
          const int ps = pt % kPSt;
          ok = mbar_wait(&p_empty[ps], empty_par(pt, kPSt), &abort_flag) && ok;
          uint32_t v[32];
          tmem_ld32(lane_addr + sb * kSCols + j * kH + hf * 32, v);
          tmem_wait_ld();
          uint32_t pk[16];
          const bool valid = (vmask >> j) & 1u;
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            const float4 m4 = *reinterpret_cast<const float4*>(mu + e);
            const float m[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
            for (int i = 0; i < 4; i += 2) {
              const float p0 = valid ? ex2_approx(fmaf(__uint_as_float(v[e + i]), c2, -m[i])) : 0.f;
              const float p1 = valid ? ex2_approx(fmaf(__uint_as_float(v[e + i + 1]), c2, -m[i + 1])) : 0.f;
              lp[e + i] += p0;
              lp[e + i + 1] += p1;
              __nv_bfloat162 b2 = __floats2bfloat162_rn(p0, p1);
              pk[(e + i) / 2] = *reinterpret_cast<uint32_t*>(&b2);
            }
          }
          uint8_t* prow_s = sP + ps * kPBytes + kk * 128;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int chunk = (hf * 4 + q) ^ (kk & 7);
            *reinterpret_cast<uint4*>(prow_s + chunk * 16) = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&p_full[ps]);
          ++pt;
        }
        fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_free[sb]);
        first = false;
        ++gi;
        if (!last) continue;
        // ---- epilogue of the item: l = sum over key lanes; o = O^T / l
        while (cons < gi) {   // every O^T update of the query
          ok = mbar_wait(&o_full[ob][cons & 1], ofw[ob][cons & 1] & 1u, &abort_flag) && ok;
          ++ofw[ob][cons & 1];
          ++cons;
        }
        fence_after_sync();
        warp_xsum32(lp, lane);
        red[hf][quad][lane] = lp[0];
        if (warp == kSmxWarp0 && lane == 0) bulk_wait_read_all();   // the previous item's output tile has left sO
        named_sync_softmax();
        if (quad == 0) {
          const int h = hf * 32 + lane;
          const float l = red[hf][0][lane] + red[hf][1][lane] + red[hf][2][lane] + red[hf][3][lane];
          l_inv[h] = l > 0.f ? 1.f / l : 0.f;
          const float lse = l > 0.f ? m_run[h] * 0.6931471805599453f + logf(l) : -INFINITY;
          if (final_out) { if (a.lse) a.lse[prow + h] = lse; }
          else a.part_lse[prow + h] = lse;
        }
        named_sync_softmax();
        uint32_t v[32];
        tmem_ld32(lane_addr + kOCol + ob * kH + hf * 32, v);
        tmem_wait_ld();
        if (final_out) {
          // o[h][d] is staged in shared memory and leaves as one 16 KB bulk copy on
          // the TMA engine, off the load/store path the producers' gathers occupy
          bf16* so = reinterpret_cast<bf16*>(sO);
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            const float4 r4 = *reinterpret_cast<const float4*>(l_inv + hf * 32 + e);
            const float r[4] = {r4.x, r4.y, r4.z, r4.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) so[(hf * 32 + e + i) * kD + kk] = __float2bfloat16_rn(__uint_as_float(v[e + i]) * r[i]);
          }
          fence_proxy_async_smem();
          named_sync_softmax();
          if (warp == kSmxWarp0 && lane == 0) {
            bulk_store_s2g(static_cast<bf16*>(a.o) + prow * kD, smem_u32(sO), kOBytes);
            bulk_commit();
          }
        } else {
#pragma unroll 4
          for (int e = 0; e < 32; ++e) {
            const int h = hf * 32 + e;
            a.part_o[(prow + h) * kD + kk] = __uint_as_float(v[e]) * l_inv[h];
          }
        }
        fence_before_sync();
        named_sync_softmax();   // l_inv / m_run are rewritten by the next item
      }
      ++n;
    }
    if (warp == kSmxWarp0 && lane == 0) bulk_wait_all();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

}  // namespace attn_tc

inline bool attn_tc_supported(int H, int D, const void* q, const void* kc, const void* vc, const void* kw,
                              const void* vw, const void* o) {
  auto al = [](const void* p) { return p == nullptr || reinterpret_cast<uintptr_t>(p) % 16 == 0; };
  return H == attn_tc::kH && D == attn_tc::kD && al(q) && al(kc) && al(vc) && al(kw) && al(vw) && al(o);
}

// Launches the tensor-core attention for all batch*T queries (nsplit slices each).
inline cudaError_t launch_attn_tc(const AttnArgs& a, int batch, cudaStream_t stream) {
  using namespace attn_tc;
  Maps m;
  const uint64_t rows_q = (uint64_t)batch * a.T * kH;
  if (!make_map_bf16_2d(&m.q, a.q, rows_q, kD, kD * 2, 64, 64)) return cudaErrorInvalidValue;
  if (!make_map_bf16_2d(&m.kw, a.kw, (uint64_t)batch * a.ring, kD, kD * 2, kTile, 64)) return cudaErrorInvalidValue;
  if (!make_map_bf16_2d(&m.vw, a.vw, (uint64_t)batch * a.ring, kD, kD * 2, kTile, 64)) return cudaErrorInvalidValue;
  // Masked keys are zero-filled with an address inside their own source; with no
  // compressed cache at all the compressed source is the window ring, so that
  // address is real memory.
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
  auto kern = a.real_kv ? attn_tc_kernel<true> : attn_tc_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, kSmem, stream>>>(m, aa, n_items);
  count_launch();
  return cudaGetLastError();
}

}  // namespace hyb
