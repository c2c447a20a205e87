// libhyb — C ABI entry points (declared and documented in include/hyb.h).
// Host side: argument checks, workspace carving, launch configuration.  The
// kernels live in the *.cuh files of this directory; this is the only
// translation unit, so the per-device status word has a single definition.
#include <cstdio>
#include <cstring>

#include "common.cuh"
#include "compress.cuh"
#include "topk.cuh"
#include "index.cuh"
#include "index_tc.cuh"
#include "hisa_tc.cuh"
#include "topk_reg.cuh"
#include "attn.cuh"
#include "attn_tc.cuh"
#include "attn_hm.cuh"

#include <type_traits>

#include <nvtx3/nvToolsExt.h>

using namespace hyb;

namespace {
// One NVTX range per C-ABI call (visible in Nsight timelines; a no-op when no
// tool is attached).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
};
}  // namespace

namespace {

constexpr size_t kAlign = 256;
inline size_t align_up(size_t x, size_t a = kAlign) { return (x + a - 1) / a * a; }
inline int round_up(int x, int m) { return (x + m - 1) / m * m; }

inline bool dtype_ok(int dtype) { return dtype == HYB_DTYPE_F32 || dtype == HYB_DTYPE_BF16; }

inline int cuda_status(cudaError_t e) { return e == cudaSuccess ? HYB_OK : HYB_ERR_CUDA; }

constexpr size_t kSmemTopkMax = 200 * 1024;  // keys staged in shared memory per row
constexpr int kHisaSlotQueries = 16;            // HISA stage 2 by kept block slot up to this many queries
constexpr size_t kScoreBudget = 64ull << 20;      // HISA: target bytes of one chunk of block scores + candidates
constexpr size_t kFlatScoreBudget = 512ull << 20; // flat: target bytes of one chunk of scores

// Queries scored per pass so that one chunk of scores stays near `budget` bytes.
// Fewer, larger chunks are faster (each chunk pays two launches and their tails)
// even where the chunk no longer fits in L2.
int default_chunk(int batch, int T, size_t row_bytes, size_t budget) {
  size_t rows = budget / (row_bytes * (size_t)batch);
  if (rows < 64) rows = 64;
  rows = rows / 64 * 64;
  return (int)(rows < (size_t)T ? rows : (size_t)T);
}

struct IndexPlan {
  int nq;        // queries per chunk (per batch)
  int ldS;       // flat: score row stride; HISA: block-score row stride
  int nb;        // HISA: blocks with a representative
  size_t off_scores, off_blk, off_ncand, off_cand, off_keys, off_list, off_work, off_nwork, off_cnt, off_fill, total;
  size_t off_cidx, off_cscore;  // flat rows longer than one register block: segment winners
  int nseg;                     // segments per row (0: single-pass selection)
  int work_cap;  // HISA grouped stage 2: work items per batch
  bool global_keys;
};

IndexPlan plan_index(int dtype, int batch, int T, int nc, int k, int mode, int block, int top_m,
                     int q_chunk) {
  (void)dtype;
  IndexPlan p{};
  if (mode == HYB_INDEX_FLAT) {
    p.ldS = round_up(nc > 0 ? nc : 1, 4);
    p.nq = q_chunk > 0 ? (q_chunk < T ? q_chunk : T) : default_chunk(batch, T, (size_t)p.ldS * 4, kFlatScoreBudget);
    p.nseg = 0;
    if (nc > kSegKeys) {
      const int nseg = (nc + kSegKeys - 1) / kSegKeys;
      if ((long long)nseg * k <= kSegKeys) p.nseg = nseg;
    }
    p.global_keys = p.nseg == 0 && (size_t)nc * 4 > kSmemTopkMax;
    size_t off = 0;
    p.off_scores = off; off += align_up((size_t)batch * p.nq * p.ldS * 4);
    p.off_keys = off;   off += p.global_keys ? align_up((size_t)batch * p.nq * p.ldS * 4) : 0;
    p.off_cidx = off;   off += p.nseg ? align_up((size_t)batch * p.nq * p.nseg * k * 4) : 0;
    p.off_cscore = off; off += p.nseg ? align_up((size_t)batch * p.nq * p.nseg * k * 4) : 0;
    p.total = off;
  } else {
    p.nb = nc / block;
    p.ldS = round_up(p.nb > 0 ? p.nb : 1, 4);
    const size_t cand = (size_t)top_m * block;
    p.nq = q_chunk > 0 ? (q_chunk < T ? q_chunk : T) : default_chunk(batch, T, cand * 4 + (size_t)p.ldS * 4, kScoreBudget);
    size_t off = 0;
    p.off_scores = off; off += align_up((size_t)batch * p.nq * p.ldS * 4);
    p.off_blk = off;    off += align_up((size_t)batch * p.nq * top_m * 4);
    p.off_ncand = off;  off += align_up((size_t)batch * p.nq * 4);
    p.off_cand = off;   off += align_up((size_t)batch * p.nq * cand * 4);
    p.work_cap = hisa_work_cap(p.nq, top_m, p.nb + 1);
    p.off_list = off;   off += align_up((size_t)batch * p.nq * top_m * 4);
    p.off_work = off;   off += align_up((size_t)batch * p.work_cap * sizeof(HgWork));
    p.off_nwork = off;  off += align_up((size_t)batch * 4);
    p.off_cnt = off;    off += align_up((size_t)batch * (p.nb + 1) * 4);
    p.off_fill = off;   off += align_up((size_t)batch * (p.nb + 1) * 4);
    p.total = off;
  }
  return p;
}

template <typename K>
cudaError_t allow_smem(K kernel, size_t bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

// Scores of query rows [i0, i0+nq) against keys (entries or block representatives):
// tensor cores for bf16 when the shape allows, CUDA cores otherwise.
template <typename T>
cudaError_t launch_scores(const void* qi, const int* q_pos, const void* keys, float* S, int batch, int T_, int i0,
                          int nq, int dI, int keys_cap, int r, int nc, int div, int ldS, cudaStream_t stream) {
  const int max_cols = nc / div;
  if (max_cols <= 0) return cudaSuccess;
  if ((nq == 1 || nq == 2) && (dI == 64 || dI == 128) && reinterpret_cast<uintptr_t>(qi) % 8 == 0 &&
      reinterpret_cast<uintptr_t>(keys) % 8 == 0) {
    // one or two rows per batch (decode): a streaming dot-product kernel
    const dim3 g((max_cols + kGvKeys - 1) / kGvKeys, batch);
    const T* q = (const T*)qi;
    const T* k = (const T*)keys;
    if constexpr (std::is_same<T, bf16>::value) {
      if (reinterpret_cast<uintptr_t>(qi) % 16 == 0 && reinterpret_cast<uintptr_t>(keys) % 16 == 0) {
        if (dI == 128) {
          if (nq == 1) scores_gemv16_kernel<16, 1><<<g, 256, 0, stream>>>(q, q_pos, k, S, T_, i0, keys_cap, r, nc, div, ldS);
          else scores_gemv16_kernel<16, 2><<<g, 256, 0, stream>>>(q, q_pos, k, S, T_, i0, keys_cap, r, nc, div, ldS);
        } else {
          if (nq == 1) scores_gemv16_kernel<8, 1><<<g, 256, 0, stream>>>(q, q_pos, k, S, T_, i0, keys_cap, r, nc, div, ldS);
          else scores_gemv16_kernel<8, 2><<<g, 256, 0, stream>>>(q, q_pos, k, S, T_, i0, keys_cap, r, nc, div, ldS);
        }
        count_launch();
        return cudaGetLastError();
      }
    }
    if (dI == 128) {
      if (nq == 1) scores_gemv_kernel<T, 4, 1><<<g, 256, 0, stream>>>(q, q_pos, k, S, T_, i0, keys_cap, r, nc, div, ldS);
      else scores_gemv_kernel<T, 4, 2><<<g, 256, 0, stream>>>(q, q_pos, k, S, T_, i0, keys_cap, r, nc, div, ldS);
    } else {
      if (nq == 1) scores_gemv_kernel<T, 2, 1><<<g, 256, 0, stream>>>(q, q_pos, k, S, T_, i0, keys_cap, r, nc, div, ldS);
      else scores_gemv_kernel<T, 2, 2><<<g, 256, 0, stream>>>(q, q_pos, k, S, T_, i0, keys_cap, r, nc, div, ldS);
    }
    count_launch();
    return cudaGetLastError();
  }
  if (std::is_same<T, bf16>::value && tc_scores_supported(dI, qi, keys))
    return launch_scores_tc(qi, q_pos, keys, S, batch, T_, i0, nq, dI, keys_cap, r, nc, div, ldS, max_cols, stream);
  dim3 g((max_cols + kSB_N - 1) / kSB_N, (nq + kSB_M - 1) / kSB_M, batch);
  scores_ffma_kernel<T><<<g, 256, 0, stream>>>((const T*)qi, q_pos, (const T*)keys, S, T_, i0, nq, dI, keys_cap,
                                               r, nc, div, ldS);
  count_launch();
  return cudaGetLastError();
}

template <typename T>
int index_topk_impl(int batch, int T_, int dI, const void* qi, const int* q_pos, const void* ic,
                    int nc, int nc_cap, int r, int k, int mode, const void* reps, int nb_cap,
                    int block, int top_m, const IndexPlan& p, int* idx, char* ws,
                    cudaStream_t stream) {
  cudaError_t e = cudaSuccess;
  float* S = reinterpret_cast<float*>(ws + p.off_scores);
  for (int i0 = 0; i0 < T_; i0 += p.nq) {
    const int nq = T_ - i0 < p.nq ? T_ - i0 : p.nq;
    if (mode == HYB_INDEX_FLAT) {
      if ((e = launch_scores<T>(qi, q_pos, ic, S, batch, T_, i0, nq, dI, nc_cap, r, nc, 1, p.ldS, stream)) !=
          cudaSuccess)
        return HYB_ERR_CUDA;
      if (nc <= 256 * kRegEPT) {
        select_flat_reg_kernel<256><<<dim3(nq, batch), 256, 0, stream>>>(S, q_pos, idx, T_, i0, nq, r, nc, k, p.ldS);
      } else if (nc <= 1024 * kRegEPT) {
        select_flat_reg_kernel<1024><<<dim3(nq, batch), 1024, 0, stream>>>(S, q_pos, idx, T_, i0, nq, r, nc, k,
                                                                           p.ldS);
      } else if (p.nseg > 0) {
        int* cidx = reinterpret_cast<int*>(ws + p.off_cidx);
        float* cscore = reinterpret_cast<float*>(ws + p.off_cscore);
        select_flat_seg_kernel<<<dim3(nq, p.nseg, batch), 1024, 0, stream>>>(S, q_pos, cidx, cscore, T_, i0, nq, r,
                                                                             nc, k, p.ldS, p.nseg);
        count_launch();
        if (p.nseg * k <= 256 * kRegEPT)
          select_flat_merge_kernel<256><<<dim3(nq, batch), 256, 0, stream>>>(q_pos, cidx, cscore, idx, T_, i0, nq, r,
                                                                              nc, k, p.nseg);
        else
          select_flat_merge_kernel<1024><<<dim3(nq, batch), 1024, 0, stream>>>(q_pos, cidx, cscore, idx, T_, i0, nq,
                                                                                r, nc, k, p.nseg);
      } else {
        const size_t smem = p.global_keys ? 0 : (size_t)nc * 4;
        if ((e = allow_smem(select_flat_kernel, smem)) != cudaSuccess) return HYB_ERR_CUDA;
        uint32_t* gkeys = p.global_keys ? reinterpret_cast<uint32_t*>(ws + p.off_keys) : nullptr;
        select_flat_kernel<<<dim3(nq, batch), kTopkThreads, smem, stream>>>(S, q_pos, idx, T_, i0, nq, r,
                                                                            nc, k, p.ldS, gkeys);
      }
      count_launch();
    } else {
      int* blk = reinterpret_cast<int*>(ws + p.off_blk);
      int* ncand = reinterpret_cast<int*>(ws + p.off_ncand);
      float* SC = reinterpret_cast<float*>(ws + p.off_cand);
      if (p.nb > 0 &&
          (e = launch_scores<T>(qi, q_pos, reps, S, batch, T_, i0, nq, dI, nb_cap, r, nc, block, p.ldS, stream)) !=
              cudaSuccess)
        return HYB_ERR_CUDA;
      if (p.nb <= 256 * kRegEPT) {
        select_blocks_reg_kernel<256><<<dim3(nq, batch), 256, 0, stream>>>(S, q_pos, blk, T_, i0, nq, r, nc, block,
                                                                          top_m, p.ldS);
      } else if (p.nb <= 1024 * kRegEPT) {
        select_blocks_reg_kernel<1024><<<dim3(nq, batch), 1024, 0, stream>>>(S, q_pos, blk, T_, i0, nq, r, nc,
                                                                            block, top_m, p.ldS);
      } else {
        const size_t smem1 = (size_t)(p.nb > 0 ? p.nb : 1) * 4;
        if ((e = allow_smem(select_blocks_kernel, smem1)) != cudaSuccess) return HYB_ERR_CUDA;
        select_blocks_kernel<<<dim3(nq, batch), kTopkThreads, smem1, stream>>>(S, q_pos, blk, T_, i0, nq, r,
                                                                               nc, block, top_m, p.ldS);
      }
      count_launch();
      if ((long long)batch * nq <= kHisaSlotQueries && dI % 4 == 0) {
        // a few queries (decode): stage 2 in one launch, one CTA per kept block
        hisa_slot_scores_kernel<T><<<dim3(top_m, nq, batch), 128, dI * 4, stream>>>(
            (const T*)qi, q_pos, (const T*)ic, blk, SC, ncand, T_, i0, nq, dI, nc_cap, r, nc, block, top_m);
        count_launch();
      } else if (hisa_grouped_supported<T>(dI, block, p.nb, qi, ic)) {
        int* list = reinterpret_cast<int*>(ws + p.off_list);
        HgWork* work = reinterpret_cast<HgWork*>(ws + p.off_work);
        int* nwork = reinterpret_cast<int*>(ws + p.off_nwork);
        int* cnt = reinterpret_cast<int*>(ws + p.off_cnt);
        int* fill = reinterpret_cast<int*>(ws + p.off_fill);
        const int nbs = p.nb + 1;
        if (i0 == 0) {
          hisa_zero_kernel<<<(batch * nbs + 255) / 256, 256, 0, stream>>>(cnt, batch * nbs);
          count_launch();
        }
        hisa_count_kernel<<<dim3((nq + 7) / 8, batch), 256, 0, stream>>>(q_pos, blk, ncand, cnt, T_, i0, nq, r, nc,
                                                                          block, top_m, nbs);
        hisa_offsets_kernel<<<batch, kHgThreads, 0, stream>>>(cnt, fill, work, nwork, nbs, p.work_cap);
        hisa_scatter_kernel<<<dim3((nq * top_m + 255) / 256, batch), 256, 0, stream>>>(blk, fill, list, nq, top_m,
                                                                                        nbs);
        count_launch();
        count_launch();
        count_launch();
        if ((e = launch_hisa_block_mma(qi, ic, list, work, nwork, SC, batch, T_, i0, nq, dI, nc_cap, top_m,
                                       p.work_cap, stream)) != cudaSuccess)
          return HYB_ERR_CUDA;
      } else {
        hisa_cand_scores_kernel<T><<<dim3(nq, batch), 256, dI * 4, stream>>>(
            (const T*)qi, q_pos, (const T*)ic, blk, SC, ncand, T_, i0, nq, dI, nc_cap, r, nc, block, top_m);
        count_launch();
      }
      const int n2 = top_m * block;
      if (n2 <= 256 * kRegEPT) {
        select_cand_reg_kernel<256><<<dim3(nq, batch), 256, 0, stream>>>(SC, ncand, blk, idx, T_, i0, nq, block,
                                                                        top_m, k);
      } else if (n2 <= 1024 * kRegEPT) {
        select_cand_reg_kernel<1024><<<dim3(nq, batch), 1024, 0, stream>>>(SC, ncand, blk, idx, T_, i0, nq, block,
                                                                          top_m, k);
      } else {
        const size_t smem2 = (size_t)n2 * 4;
        if ((e = allow_smem(select_cand_kernel, smem2)) != cudaSuccess) return HYB_ERR_CUDA;
        select_cand_kernel<<<dim3(nq, batch), kTopkThreads, smem2, stream>>>(SC, ncand, blk, idx, T_, i0, nq,
                                                                             block, top_m, k);
      }
      count_launch();
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return HYB_ERR_CUDA;
  }
  return HYB_OK;
}

// Streaming multiprocessors of the current device (148 on B200; also the value
// used where no device is visible, so that workspace sizes can be queried on a
// host without a GPU).
int sm_count() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) {
    cudaGetLastError();
    return 148;
  }
  return sms;
}

int attn_splits(int mode, int batch, int T, int n_keys_max) {
  if (mode != HYB_ATTN_DECODE) return 1;
  // a slice is one latency chain of the kernel, and the partial outputs and their
  // merge cost more than a chain: split only while fewer than half the SMs would
  // have a query (batch 64 at 128K: no split, CSA 0.025 ms against 0.035 with two
  // slices and 0.047 with one per key tile), at least 64 keys per split
  const int ctas = batch * T;
  int ns = sm_count() / (2 * ctas);
  const int cap = (n_keys_max + 63) / 64;
  if (ns > cap) ns = cap;
  if (ns < 1) ns = 1;
  if (ns > 64) ns = 64;
  return ns;
}

}  // namespace

extern "C" {

const char* hyb_status_string(int status) {
  switch (status) {
    case HYB_OK: return "HYB_OK";
    case HYB_ERR_INVALID_ARG: return "HYB_ERR_INVALID_ARG: invalid argument";
    case HYB_ERR_UNSUPPORTED: return "HYB_ERR_UNSUPPORTED: dtype, size or alignment not supported";
    case HYB_ERR_WORKSPACE: return "HYB_ERR_WORKSPACE: workspace missing or too small";
    case HYB_ERR_CUDA: return "HYB_ERR_CUDA: CUDA launch or runtime call failed";
    case HYB_ERR_TIMEOUT: return "HYB_ERR_TIMEOUT: a bounded device wait gave up";
    case HYB_ERR_DEVICE_CHECK: return "HYB_ERR_DEVICE_CHECK: a device-side index or size check failed";
    default: return "HYB_ERR_UNKNOWN";
  }
}

int hyb_abi_version(void) { return 100; }

unsigned long long hyb_kernel_launches(void) { return launch_counter().load(); }

int hyb_get_device_status(hyb_stream_t stream, int* status) {
  if (!status) return HYB_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int host = 0;
  const int zero = 0;
  if (cudaStreamSynchronize(s) != cudaSuccess) return HYB_ERR_CUDA;
  if (cudaMemcpyFromSymbolAsync(&host, g_status, sizeof(int), 0, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return HYB_ERR_CUDA;
  if (cudaMemcpyToSymbolAsync(g_status, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return HYB_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return HYB_ERR_CUDA;
  *status = host;
  return HYB_OK;
}

int hyb_compress(int dtype, int batch, int L, int D, int dI, const void* xk, const void* xv,
                 const void* xi, const float* logits, const float* bias, int r, int overlap,
                 int j_begin, int j_end, void* kc, void* vc, void* ic, int nc_cap,
                 hyb_stream_t stream) {
  NvtxRange nvtx_range("hyb_compress");
  if (!dtype_ok(dtype)) return HYB_ERR_UNSUPPORTED;
  if (batch < 0 || L < 0 || D <= 0 || r < 1 || j_begin < 0 || j_end < j_begin || nc_cap < j_end)
    return HYB_ERR_INVALID_ARG;
  if ((long long)j_end * r > L) return HYB_ERR_INVALID_ARG;
  if (!xk || !xv || !logits || !bias || !kc || !vc) return HYB_ERR_INVALID_ARG;
  if (xi && (!ic || dI <= 0)) return HYB_ERR_INVALID_ARG;
  const int span = overlap ? 2 * r : r;
  if (span > kMaxSpan || D % 4 != 0 || (xi && dI % 4 != 0)) return HYB_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = dtype == HYB_DTYPE_F32
      ? launch_compress<float>(batch, L, D, dI, xk, xv, xi, logits, bias, r, overlap ? 1 : 0, j_begin,
                               j_end, kc, vc, ic, nc_cap, s)
      : launch_compress<bf16>(batch, L, D, dI, xk, xv, xi, logits, bias, r, overlap ? 1 : 0, j_begin,
                              j_end, kc, vc, ic, nc_cap, s);
  return cuda_status(e);
}

int hyb_compress_pc(int dtype, int batch, int L, int D, int dI, const void* xk, const void* xv, const void* xi,
                    const float* z_kv, const float* bias_kv, const float* z_i, const float* bias_i, int r,
                    int overlap, int j_begin, int j_end, void* kc, void* vc, void* ic, int nc_cap,
                    hyb_stream_t stream) {
  NvtxRange nvtx_range("hyb_compress_pc");
  if (!dtype_ok(dtype)) return HYB_ERR_UNSUPPORTED;
  if (batch < 0 || L < 0 || D <= 0 || r < 1 || j_begin < 0 || j_end < j_begin || nc_cap < j_end)
    return HYB_ERR_INVALID_ARG;
  if ((long long)j_end * r > L) return HYB_ERR_INVALID_ARG;
  if (!xk || !xv || !z_kv || !bias_kv || !kc || !vc) return HYB_ERR_INVALID_ARG;
  if (xi && (!ic || !z_i || !bias_i || dI <= 0)) return HYB_ERR_INVALID_ARG;
  auto al = [](const void* p) { return p == nullptr || reinterpret_cast<uintptr_t>(p) % 16 == 0; };
  const int span = overlap ? 2 * r : r;
  if (span > kMaxSpan || D % 4 != 0 || (xi && dI % 4 != 0) || !al(z_kv) || !al(bias_kv) || !al(z_i) || !al(bias_i))
    return HYB_ERR_UNSUPPORTED;
  const int n = j_end - j_begin;
  if (n == 0 || batch == 0) return HYB_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const dim3 grid((n + kCompressWarps - 1) / kCompressWarps, batch);
  if (dtype == HYB_DTYPE_F32)
    compress_pc_kernel<float><<<grid, kCompressWarps * 32, 0, s>>>(
        (const float*)xk, (const float*)xv, (const float*)xi, z_kv, bias_kv, z_i, bias_i, (float*)kc, (float*)vc,
        (float*)ic, L, D, dI, r, overlap ? 1 : 0, j_begin, j_end, nc_cap);
  else
    compress_pc_kernel<bf16><<<grid, kCompressWarps * 32, 0, s>>>(
        (const bf16*)xk, (const bf16*)xv, (const bf16*)xi, z_kv, bias_kv, z_i, bias_i, (bf16*)kc, (bf16*)vc,
        (bf16*)ic, L, D, dI, r, overlap ? 1 : 0, j_begin, j_end, nc_cap);
  count_launch();
  return cuda_status(cudaGetLastError());
}

int hyb_decode_append(int dtype, int batch, int D, int dI, const void* xk_new, const void* xv_new,
                      const void* xi_new, const float* z_new, const int* pos, void* kw, void* vw, void* iw,
                      float* zw, int ring, const float* bias_csa, int r_csa, int overlap, void* kc, void* vc,
                      void* ic, int nc_cap, const float* bias_hca, int r_hca, void* kc_hca, void* vc_hca,
                      int nch_cap, int block, void* reps, int nb_cap, hyb_stream_t stream) {
  NvtxRange nvtx_range("hyb_decode_append");
  if (!dtype_ok(dtype)) return HYB_ERR_UNSUPPORTED;
  if (batch < 0 || D <= 0 || ring < 1) return HYB_ERR_INVALID_ARG;
  if (batch == 0) return HYB_OK;
  if (!xk_new || !xv_new || !z_new || !pos || !kw || !vw || !zw) return HYB_ERR_INVALID_ARG;
  if (xi_new && (!iw || dI <= 0)) return HYB_ERR_INVALID_ARG;
  if (D % 4 != 0 || (xi_new && dI % 4 != 0)) return HYB_ERR_UNSUPPORTED;
  if (bias_csa) {
    const int span = overlap ? 2 * r_csa : r_csa;
    if (r_csa < 1 || nc_cap < 0 || !kc || !vc || (xi_new && !ic)) return HYB_ERR_INVALID_ARG;
    if (span > ring || span > kMaxSpan) return HYB_ERR_UNSUPPORTED;
    if (reps && (!xi_new || block < 1 || nb_cap < 0)) return HYB_ERR_INVALID_ARG;
  }
  if (bias_hca) {
    if (r_hca < 1 || nch_cap < 0 || !kc_hca || !vc_hca) return HYB_ERR_INVALID_ARG;
    if (r_hca > ring || r_hca > kMaxSpan) return HYB_ERR_UNSUPPORTED;
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const void* ici = bias_csa ? ic : nullptr;
  void* rp = bias_csa ? reps : nullptr;
  if (dtype == HYB_DTYPE_F32) {
    decode_append_kernel<float><<<batch, 32, 0, s>>>(
        (const float*)xk_new, (const float*)xv_new, (const float*)xi_new, z_new, pos, (float*)kw, (float*)vw,
        (float*)(xi_new ? iw : nullptr), zw, ring, D, dI, bias_csa, r_csa, overlap ? 1 : 0, (float*)kc, (float*)vc,
        (float*)ici, nc_cap, bias_hca, r_hca, (float*)kc_hca, (float*)vc_hca, nch_cap, block, (float*)rp, nb_cap);
  } else {
    decode_append_kernel<bf16><<<batch, 32, 0, s>>>(
        (const bf16*)xk_new, (const bf16*)xv_new, (const bf16*)xi_new, z_new, pos, (bf16*)kw, (bf16*)vw,
        (bf16*)(xi_new ? iw : nullptr), zw, ring, D, dI, bias_csa, r_csa, overlap ? 1 : 0, (bf16*)kc, (bf16*)vc,
        (bf16*)ici, nc_cap, bias_hca, r_hca, (bf16*)kc_hca, (bf16*)vc_hca, nch_cap, block, (bf16*)rp, nb_cap);
  }
  count_launch();
  return cuda_status(cudaGetLastError());
}

int hyb_block_reps(int dtype, int batch, int dI, const void* ic, int nc_cap, int block, int g_begin,
                   int g_end, void* reps, int nb_cap, hyb_stream_t stream) {
  NvtxRange nvtx_range("hyb_block_reps");
  if (!dtype_ok(dtype)) return HYB_ERR_UNSUPPORTED;
  if (batch < 0 || dI <= 0 || block < 1 || g_begin < 0 || g_end < g_begin || g_end > nb_cap ||
      (long long)g_end * block > nc_cap)
    return HYB_ERR_INVALID_ARG;
  if (!ic || !reps) return HYB_ERR_INVALID_ARG;
  if (dI % 4 != 0) return HYB_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = dtype == HYB_DTYPE_F32
      ? launch_block_reps<float>(batch, dI, ic, nc_cap, block, g_begin, g_end, reps, nb_cap, s)
      : launch_block_reps<bf16>(batch, dI, ic, nc_cap, block, g_begin, g_end, reps, nb_cap, s);
  return cuda_status(e);
}

size_t hyb_index_topk_workspace_size(int dtype, int batch, int T, int nc, int dI, int k, int mode,
                                     int block, int top_m, int q_chunk) {
  (void)dI;
  if (batch <= 0 || T <= 0 || nc < 0 || k < 1) return 0;
  if (mode == HYB_INDEX_HISA && (block < 1 || top_m < 1)) return 0;
  return plan_index(dtype, batch, T, nc, k, mode, block, top_m, q_chunk).total;
}

int hyb_index_topk(int dtype, int batch, int T, int dI, const void* qi, const int* q_pos,
                   const void* ic, int nc, int nc_cap, int r, int k, int mode, const void* reps,
                   int nb_cap, int block, int top_m, int q_chunk, int* idx, void* ws,
                   size_t ws_bytes, hyb_stream_t stream) {
  NvtxRange nvtx_range("hyb_index_topk");
  if (!dtype_ok(dtype)) return HYB_ERR_UNSUPPORTED;
  if (mode != HYB_INDEX_FLAT && mode != HYB_INDEX_HISA) return HYB_ERR_INVALID_ARG;
  if (batch < 0 || T < 0 || dI <= 0 || nc < 0 || nc_cap < nc || r < 1 || k < 1 || q_chunk < 0)
    return HYB_ERR_INVALID_ARG;
  if (batch == 0 || T == 0) return HYB_OK;
  if (!qi || !q_pos || !ic || !idx) return HYB_ERR_INVALID_ARG;
  if (dI % 4 != 0) return HYB_ERR_UNSUPPORTED;
  if (mode == HYB_INDEX_HISA) {
    if (block < 1 || top_m < 1 || !reps || nb_cap < nc / block) return HYB_ERR_INVALID_ARG;
    if ((size_t)top_m * block * 4 > kSmemTopkMax || (size_t)(nc / block) * 4 > kSmemTopkMax)
      return HYB_ERR_UNSUPPORTED;
  }
  const IndexPlan p = plan_index(dtype, batch, T, nc, k, mode, block, top_m, q_chunk);
  if (!ws || ws_bytes < p.total || (reinterpret_cast<uintptr_t>(ws) % kAlign) != 0) return HYB_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  char* w = static_cast<char*>(ws);
  return dtype == HYB_DTYPE_F32
      ? index_topk_impl<float>(batch, T, dI, qi, q_pos, ic, nc, nc_cap, r, k, mode, reps, nb_cap, block,
                               top_m, p, idx, w, s)
      : index_topk_impl<bf16>(batch, T, dI, qi, q_pos, ic, nc, nc_cap, r, k, mode, reps, nb_cap, block,
                              top_m, p, idx, w, s);
}

size_t hyb_attn_fwd_workspace_size(int dtype, int batch, int T, int H, int D, int k, int nc, int W,
                                   int mode) {
  (void)dtype;
  if (batch <= 0 || T <= 0 || H <= 0 || D <= 0) return 0;
  const int n_keys = (k > 0 ? k : nc) + W;
  const int ns = attn_splits(mode & ~HYB_ATTN_REAL_KV, batch, T, n_keys);
  if (ns <= 1) return 0;
  const size_t rows = (size_t)batch * T * ns * H;
  return align_up(rows * D * 4) + align_up(rows * 4);
}

}  // extern "C"

namespace {

int attn_fwd_impl(int dtype, int batch, int T, int H, int D, const void* q, const int* q_pos,
                  const void* kc, const void* vc, int nc, int nc_cap, int r, const int* idx, int k,
                  const void* kw, const void* vw, int ring, int W, float scale, void* o, float* lse,
                  int mode, void* ws, size_t ws_bytes, hyb_stream_t stream, unsigned long long wait_ns,
                  int drop_arrival) {
  if (!dtype_ok(dtype)) return HYB_ERR_UNSUPPORTED;
  const bool real_kv = (mode & HYB_ATTN_REAL_KV) != 0;
  mode &= ~HYB_ATTN_REAL_KV;
  if (mode != HYB_ATTN_PREFILL && mode != HYB_ATTN_DECODE) return HYB_ERR_INVALID_ARG;
  if (batch < 0 || T < 0 || H <= 0 || D <= 0 || nc < 0 || (!real_kv && nc_cap < nc) || r < 1 || W < 0 ||
      (idx && k < 1) || ring < 1 || ring < W || (real_kv && !idx))
    return HYB_ERR_INVALID_ARG;
  if (batch == 0 || T == 0) return HYB_OK;
  if (!q || !q_pos || !kw || !vw || !o || (!real_kv && (nc > 0) && (!kc || !vc))) return HYB_ERR_INVALID_ARG;
  const bool tc = dtype == HYB_DTYPE_BF16 && attn_tc_supported(H, D, q, real_kv ? nullptr : kc,
                                                                real_kv ? nullptr : vc, kw, vw, o);
  if (!attn_ffma_supported(H, D) && !tc) return HYB_ERR_UNSUPPORTED;
  if (real_kv && (!tc || (long long)k * r > (1 << 30))) return HYB_ERR_UNSUPPORTED;   // tensor-core kernel only
  if (real_kv) kc = vc = nullptr;   // the keys come from the ring
  const int n_keys = (idx ? k : nc) + W;
  int ns = attn_splits(mode, batch, T, n_keys);
  if (ns > 1 && tc) {
    // the tensor-core kernel splits a query's keys at 128-key tiles: no more slices
    // than tiles, and no empty slice
    const int n_comp = idx ? (real_kv ? k * r : k) : nc;
    const int tiles = (n_comp + attn_tc::kTile - 1) / attn_tc::kTile + (W + attn_tc::kTile - 1) / attn_tc::kTile;
    if (ns > tiles) ns = tiles;
    const int per = (tiles + ns - 1) / ns;
    ns = (tiles + per - 1) / per;
  }
  AttnArgs a{q, q_pos, kc, vc, nc, nc_cap, r, idx, k, kw, vw, ring, W, scale, o, lse,
             nullptr, nullptr, T, H, D, ns, real_kv ? 1 : 0, wait_ns, drop_arrival};
  if (ns > 1) {
    const size_t rows = (size_t)batch * T * ns * H;
    const size_t need = align_up(rows * D * 4) + align_up(rows * 4);
    if (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) % kAlign) != 0) return HYB_ERR_WORKSPACE;
    a.part_o = static_cast<float*>(ws);
    a.part_lse = reinterpret_cast<float*>(static_cast<char*>(ws) + align_up(rows * D * 4));
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (dtype == HYB_DTYPE_F32) {
    if ((e = launch_attn_ffma<float>(a, batch, s)) != cudaSuccess) return HYB_ERR_CUDA;
    if (ns > 1) { attn_merge_kernel<float><<<dim3(batch * T, H), 128, 0, s>>>(a); count_launch(); }
  } else {
    if (tc)
      e = real_kv ? launch_attn_tc(a, batch, s) : launch_attn_hm(a, batch, s);
    else
      e = launch_attn_ffma<bf16>(a, batch, s);
    if (e != cudaSuccess) return HYB_ERR_CUDA;
    if (ns > 1) { attn_merge_kernel<bf16><<<dim3(batch * T, H), 128, 0, s>>>(a); count_launch(); }
  }
  return cuda_status(cudaGetLastError());
}

}  // namespace

extern "C" {

int hyb_attn_fwd(int dtype, int batch, int T, int H, int D, const void* q, const int* q_pos,
                 const void* kc, const void* vc, int nc, int nc_cap, int r, const int* idx, int k,
                 const void* kw, const void* vw, int ring, int W, float scale, void* o, float* lse,
                 int mode, void* ws, size_t ws_bytes, hyb_stream_t stream) {
  NvtxRange nvtx_range("hyb_attn_fwd");
  return attn_fwd_impl(dtype, batch, T, H, D, q, q_pos, kc, vc, nc, nc_cap, r, idx, k, kw, vw, ring, W, scale, o,
                       lse, mode, ws, ws_bytes, stream, sm100::kWaitNs, 0);
}

int hyb_attn_fwd_wait_test(int dtype, int batch, int T, int H, int D, const void* q, const int* q_pos,
                           const void* kc, const void* vc, int nc, int nc_cap, int r, const int* idx, int k,
                           const void* kw, const void* vw, int ring, int W, float scale, void* o, float* lse,
                           int mode, void* ws, size_t ws_bytes, hyb_stream_t stream, unsigned long long wait_ns,
                           int drop_arrival) {
  NvtxRange nvtx_range("hyb_attn_fwd_wait_test");
  if (wait_ns == 0 || wait_ns > sm100::kWaitNs) return HYB_ERR_INVALID_ARG;
  // only the heads-in-M tensor-core kernel has the hook
  if (dtype != HYB_DTYPE_BF16 || H != attn_hm::kH || D != attn_hm::kD || (mode & HYB_ATTN_REAL_KV))
    return HYB_ERR_UNSUPPORTED;
  return attn_fwd_impl(dtype, batch, T, H, D, q, q_pos, kc, vc, nc, nc_cap, r, idx, k, kw, vw, ring, W, scale, o,
                       lse, mode, ws, ws_bytes, stream, wait_ns, drop_arrival ? 1 : 0);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Flat indexer without caller-provided scratch.
//
// Some callers cannot hand the library device memory: an inference engine that
// gives the whole of HBM to its own pool allocator (cudaMalloc then fails, or
// fragments the pool), or a plugin running inside a host framework that owns
// all device allocations.  hyb_index_topk_noalloc serves them: its scores live
// in the fixed array below, which every GPU that loads this library holds until
// the process exits.  All calls on a device share it and it keeps the previous
// call's contents; nothing in it needs to start at zero (every score is written
// before it is read), but two calls whose kernels overlap on the GPU (different
// streams, no ordering between them) race on it.
constexpr size_t kNoAllocScratchBytes = 16u << 20;   // 16 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
// Device address of the scratch array in the calling thread's current context.
// The host-side symbol is not a device address, and the address can change when
// the library's module is loaded again (after cudaDeviceReset, or in another
// context of the same device), so it is looked up on every call: a host-side
// table lookup that allocates nothing.
int noalloc_scratch(void** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return HYB_ERR_CUDA;
  *out = p;
  return HYB_OK;
}
}  // namespace

extern "C" int hyb_index_topk_noalloc(int dtype, int batch, int T, int dI, const void* qi, const int* q_pos,
                                      const void* ic, int nc, int nc_cap, int r, int k, int* idx,
                                      hyb_stream_t stream) {
  NvtxRange nvtx_range("hyb_index_topk_noalloc");
  if (!dtype_ok(dtype)) return HYB_ERR_UNSUPPORTED;
  if (batch < 0 || T < 0 || dI <= 0 || nc < 0 || nc_cap < nc || r < 1 || k < 1) return HYB_ERR_INVALID_ARG;
  if (batch == 0 || T == 0) return HYB_OK;
  if (!qi || !q_pos || !ic || !idx) return HYB_ERR_INVALID_ARG;
  if (dI % 4 != 0) return HYB_ERR_UNSUPPORTED;
  // one row of scores per batch entry must fit, and rows must not need the
  // global-memory key buffer of the longest-row path
  const size_t row_bytes = (size_t)round_up(nc > 0 ? nc : 1, 4) * 4;
  if (nc > 1024 * kRegEPT || row_bytes * (size_t)batch > kNoAllocScratchBytes) return HYB_ERR_UNSUPPORTED;
  int nq = (int)(kNoAllocScratchBytes / (row_bytes * (size_t)batch));
  if (nq > T) nq = T;
  const IndexPlan p = plan_index(dtype, batch, T, nc, k, HYB_INDEX_FLAT, 0, 0, nq);
  if (p.total > kNoAllocScratchBytes || p.global_keys) return HYB_ERR_UNSUPPORTED;
  void* ws = nullptr;
  const int st = noalloc_scratch(&ws);
  if (st != HYB_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  char* w = static_cast<char*>(ws);
  return dtype == HYB_DTYPE_F32
      ? index_topk_impl<float>(batch, T, dI, qi, q_pos, ic, nc, nc_cap, r, k, HYB_INDEX_FLAT, nullptr, 0, 0, 0, p,
                               idx, w, s)
      : index_topk_impl<bf16>(batch, T, dI, qi, q_pos, ic, nc, nc_cap, r, k, HYB_INDEX_FLAT, nullptr, 0, 0, 0, p,
                              idx, w, s);
}
