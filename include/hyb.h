/*
 * hyb.h — C ABI of libhyb: the forward pass of one hybrid compressed attention
 * layer (CSA: compressed + sparse; HCA: heavily compressed + dense) on one
 * NVIDIA B200 (sm_100a).
 *
 * The method is described on public pages only:
 *  - "Hybrid Attention" explainer (process-cxr.github.io), section
 *    "DeepSeek V4 中的定义": CSA compresses the KV cache along the sequence and
 *    applies sparse attention; HCA compresses harder and attends densely.
 *  - HCA article (daiw.net, "前代 · HCA：128 倍压缩后再做稠密注意力"), section
 *    "怎么压" (How it is compressed) and the CSA/HCA table: softmax-weighted
 *    pooling with a learnable positional bias, r = 128 without overlap (CSA:
 *    r = 4, overlapping), shared-KV (MQA) attention, a 128-token sliding window.
 *  - HISA write-up (my.qihongyi.cn, "DeepSeek速度狂飙4倍还不丢精度"), sections
 *    01, 02 and 05, Fig. 2: flat top-k indexer; two-stage block/token indexer.
 *  - trdm.cn news 749237, section 2.1: CSA = 4:1 compression + indexer top-k +
 *    128-token window; HCA = 128:1 compression + dense attention.
 *
 * Conventions for every call:
 *  - All tensor pointers are DEVICE pointers owned by the caller; the library
 *    allocates nothing, keeps no pointer after returning and never
 *    synchronises (except hyb_get_device_status).  Work is enqueued on
 *    `stream` (a cudaStream_t; NULL = legacy default stream).
 *  - Tensors are dense row-major with the batch dimension outermost; shapes
 *    are given per argument.  `dtype` is HYB_DTYPE_F32 or HYB_DTYPE_BF16 and
 *    applies to every non-fp32-typed tensor of the call (logits, bias and lse
 *    are always fp32; positions and indices int32).
 *  - Positions are absolute token positions (0-based).  Compressed entry j
 *    covers raw tokens [(j-1)r, (j+1)r) (overlap = 1, clipped at 0) or
 *    [jr, (j+1)r) (overlap = 0) and is visible to the query at position t iff
 *    j < floor((t+1)/r) (its last token is at or before t).
 *  - Return value: HYB_OK, or an error code from argument checks done on the
 *    host before anything is launched (nothing is enqueued on error), or
 *    HYB_ERR_CUDA when a launch failed.  Errors found by the kernels
 *    themselves (an index out of range, a bounded wait that gave up) are
 *    recorded in a per-device status word, read and cleared by
 *    hyb_get_device_status.  No call traps, asserts or spins without bound.
 *  - Calls are thread-safe and keep no state between calls other than the
 *    per-device status word.  One exception: hyb_index_topk_noalloc keeps
 *    its scores in one fixed device array per GPU, shared by all of its calls
 *    on that GPU, so two of its calls must never run on one GPU at the same
 *    time (see its comment).
 */
#ifndef HYB_H_
#define HYB_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* hyb_stream_t; /* same type as cudaStream_t */

enum {
  HYB_OK = 0,
  HYB_ERR_INVALID_ARG = 1,  /* null pointer, negative or inconsistent size    */
  HYB_ERR_UNSUPPORTED = 2,  /* dtype, size or alignment outside what is built */
  HYB_ERR_WORKSPACE = 3,    /* workspace missing or smaller than required     */
  HYB_ERR_CUDA = 4,         /* a CUDA launch or runtime call failed           */
  HYB_ERR_TIMEOUT = 5,      /* device: a bounded wait gave up (status word)   */
  HYB_ERR_DEVICE_CHECK = 6  /* device: an index or size check failed (status) */
};

enum { HYB_DTYPE_F32 = 0, HYB_DTYPE_BF16 = 1 };
enum { HYB_INDEX_FLAT = 0, HYB_INDEX_HISA = 1 };
enum { HYB_ATTN_PREFILL = 0, HYB_ATTN_DECODE = 1 };
/* Flag OR-ed into the attention mode: the "real K/V" reading of CSA (see hyb_attn_fwd). */
enum { HYB_ATTN_REAL_KV = 2 };

/* Human-readable name of a status code.  Never NULL. */
const char* hyb_status_string(int status);

/* ABI version of this header (major*100 + minor). */
int hyb_abi_version(void);

/* Number of kernels this library has launched in this process (all devices),
 * counted on the host at launch time: launch accounting for benchmarks. */
unsigned long long hyb_kernel_launches(void);

/*
 * Reads the calling device's status word after synchronising `stream`, stores
 * it in *status (HYB_OK when no kernel reported an error since the last read)
 * and clears it.  Returns HYB_ERR_CUDA if the copy or synchronisation failed.
 */
int hyb_get_device_status(hyb_stream_t stream, int* status);

/*
 * S1 — sequence-axis compression (HCA article, section "怎么压"; CSA/HCA table;
 * trdm.cn 2.1).  For every batch b and entry j in [j_begin, j_end):
 *   w_i = softmax over the window of (logits[b, i] + bias[p]),
 *   p = i - window_start(j) (position in the unclipped window),
 *   kc[b, j] = sum_i w_i xk[b, i];  vc[b, j] = sum_i w_i xv[b, i];
 *   ic[b, j] = sum_i w_i xi[b, i]  (when xi != NULL).
 * The weights are computed in fp32 and the sums accumulated in fp32.
 *   xk, xv  [batch, L, D]       xi [batch, L, dI] or NULL (then ic unused)
 *   logits  [batch, L] fp32     bias [2r] (overlap = 1) or [r] (overlap = 0) fp32
 *   kc, vc  [batch, nc_cap, D]  ic [batch, nc_cap, dI]
 * Requires 0 <= j_begin <= j_end <= nc_cap, j_end * r <= L (whole windows
 * only), r >= 1, window length (2r or r) <= 256, D and dI multiples of 4.
 */
int hyb_compress(int dtype, int batch, int L, int D, int dI,
                 const void* xk, const void* xv, const void* xi,
                 const float* logits, const float* bias, int r, int overlap,
                 int j_begin, int j_end,
                 void* kc, void* vc, void* ic, int nc_cap,
                 hyb_stream_t stream);

/*
 * S1 with per-channel compression weights (the other reading of "compression
 * weights", HCA article, section "怎么压"): channel c of entry j is
 * sum_i w[i, c] x[i, c], w[., c] = softmax over the window's in-range tokens of
 * (z[i, c] + bias[p, c]), p the position in the unclipped window.  K and V use
 * z_kv [batch, L, D] and bias_kv [span, D] (fp32); the indexer keys (xi, nullable)
 * use z_i [batch, L, dI] and bias_i [span, dI].  Windows, layouts, capacities and
 * requirements as for hyb_compress; logits and biases 16-byte aligned.
 */
int hyb_compress_pc(int dtype, int batch, int L, int D, int dI,
                    const void* xk, const void* xv, const void* xi,
                    const float* z_kv, const float* bias_kv, const float* z_i, const float* bias_i,
                    int r, int overlap, int j_begin, int j_end,
                    void* kc, void* vc, void* ic, int nc_cap, hyb_stream_t stream);

/*
 * HISA stage-1 representatives (HISA write-up, section 02, stage 1: each block
 * of `block` entries is summarised by one pooled vector; the mean is used).
 * For blocks g in [g_begin, g_end): reps[b, g] = mean of ic[b, g*block ..
 * (g+1)*block - 1], accumulated in fp32 and stored in `dtype`.
 *   ic [batch, nc_cap, dI]   reps [batch, nb_cap, dI]
 * Requires g_end * block <= nc_cap, g_end <= nb_cap, dI multiple of 4.
 */
int hyb_block_reps(int dtype, int batch, int dI, const void* ic, int nc_cap,
                   int block, int g_begin, int g_end, void* reps, int nb_cap,
                   hyb_stream_t stream);

/*
 * Decode-step state update, fused (the step just before index + attend when
 * serving: append the raw token to the window ring, emit a compressed entry
 * every r tokens, refresh the HISA representative every `block` entries; HCA
 * article, section "怎么压", and HISA write-up, section 02, stage 1).
 * For each sequence b the new token is at position t = pos[b] (device int32):
 *  - xk_new, xv_new [batch, D], xi_new [batch, dI] (nullable), z_new [batch]
 *    (its compression logit) are written to slot t mod ring of the rings
 *    kw, vw [batch, ring, D], iw [batch, ring, dI] (required with xi_new) and
 *    zw [batch, ring] fp32 (the rings also serve as the attention window ring);
 *  - when t + 1 is a multiple of r_csa (bias_csa non-null), CSA entry
 *    j = (t+1)/r_csa - 1 of kc, vc [batch, nc_cap, D] and ic [batch, nc_cap, dI]
 *    is written, pooled exactly as hyb_compress would from the full sequence;
 *    when moreover j + 1 is a multiple of `block` (reps non-null), reps[b, g]
 *    (g = (j+1)/block - 1) of reps [batch, nb_cap, dI] is recomputed as
 *    hyb_block_reps would;
 *  - when t + 1 is a multiple of r_hca (bias_hca non-null), HCA entry
 *    (t+1)/r_hca - 1 of kc_hca, vc_hca [batch, nch_cap, D] is written.
 * Requires ring >= the window lengths (2 r_csa with overlap, else r_csa; r_hca),
 * windows <= 256, D and dI multiples of 4.  An entry index past its capacity or
 * a negative position sets HYB_ERR_DEVICE_CHECK (read with hyb_get_device_status).
 * Results are bit-identical to hyb_compress / hyb_block_reps on the same tokens.
 */
int hyb_decode_append(int dtype, int batch, int D, int dI,
                      const void* xk_new, const void* xv_new, const void* xi_new, const float* z_new,
                      const int* pos, void* kw, void* vw, void* iw, float* zw, int ring,
                      const float* bias_csa, int r_csa, int overlap, void* kc, void* vc, void* ic,
                      int nc_cap, const float* bias_hca, int r_hca, void* kc_hca, void* vc_hca,
                      int nch_cap, int block, void* reps, int nb_cap, hyb_stream_t stream);

/*
 * S2 — indexer and top-k selection (HISA write-up, sections 01 and 02; the
 * output contract of section 05 step 3: k entry indices per query).
 * Query (b, i) at position t = q_pos[b, i] sees entries j < V = min(floor((t+1)/r), nc);
 * its score for entry j is qi[b, i] . ic[b, j] (fp32 accumulation).
 *  mode HYB_INDEX_FLAT: keep the k best of the V entries.
 *  mode HYB_INDEX_HISA: full visible blocks g < floor(V/block) are scored by
 *    qi . reps[b, g]; the partial block (when V mod block != 0) is always kept;
 *    the best full blocks fill the remaining top_m slots; then the k best of
 *    the visible entries of the kept blocks are selected.
 * Ties go to the lower index (entries and blocks).  The idx row holds the
 * selected entries in ascending order followed by -1 when fewer than k exist.
 *   qi [batch, T, dI]   q_pos [batch, T] int32   ic [batch, nc_cap, dI]
 *   reps [batch, nb_cap, dI] with nb_cap >= floor(nc/block) (HISA only)
 *   idx [batch, T, k] int32
 * `q_chunk` is the number of queries scored per pass (a scheduling choice;
 * results do not depend on it; 0 = library default: about 512 MiB of fp32
 * scores per pass for FLAT, about 64 MiB of block scores and candidates for
 * HISA; a smaller q_chunk shrinks the workspace).  Scratch comes from
 * `ws` (device memory, 256-byte aligned) of at least
 * hyb_index_topk_workspace_size(...) bytes.
 */
size_t hyb_index_topk_workspace_size(int dtype, int batch, int T, int nc, int dI, int k,
                                     int mode, int block, int top_m, int q_chunk);
int hyb_index_topk(int dtype, int batch, int T, int dI,
                   const void* qi, const int* q_pos,
                   const void* ic, int nc, int nc_cap, int r, int k, int mode,
                   const void* reps, int nb_cap, int block, int top_m, int q_chunk,
                   int* idx, void* ws, size_t ws_bytes, hyb_stream_t stream);

/*
 * Flat indexer with no caller-provided scratch (no counterpart on the pages:
 * this is an interface for callers, not part of the method).
 *
 * Same arguments and results as hyb_index_topk in HYB_INDEX_FLAT mode, minus
 * the workspace.  It is for callers that cannot allocate device memory for the
 * library, such as an inference engine whose pool allocator owns all of HBM or
 * a plugin whose host framework does every device allocation itself.  The
 * library allocates nothing here either: the scores go to a 16 MiB array that
 * is part of the library's device image, so every GPU that loads libhyb holds
 * those 16 MiB until the process exits.
 *  - Every call looks up the array's device address in the current context
 *    (a host-side lookup; the address changes if the library's device code is
 *    loaded again, e.g. after cudaDeviceReset).  The first call on a device
 *    may load the library's device code; make it before any stream capture.
 *  - All calls on a device share the array.  Calls whose kernels may run at the
 *    same time on that device (different streams without ordering) race on it
 *    and must not be issued.
 *  - Returns HYB_ERR_UNSUPPORTED when batch * round_up(nc, 4) * 4 bytes exceed
 *    the 16 MiB array or nc > 32768; queries are scored in chunks that fit.
 */
int hyb_index_topk_noalloc(int dtype, int batch, int T, int dI,
                           const void* qi, const int* q_pos,
                           const void* ic, int nc, int nc_cap, int r, int k,
                           int* idx, hyb_stream_t stream);

/*
 * S3 + S4 — shared-KV attention with a sliding window (HCA article, section
 * "怎么压": MQA over all compressed entries (HCA) plus a 128-token window branch,
 * as in CSA; trdm.cn 2.1: CSA attends the indexer's top-k plus the window).
 * For query (b, i) at t = q_pos[b, i] and every head h, the key set is
 *   { compressed entries idx[b, i, :] >= 0 }          (idx != NULL, CSA)
 *   { compressed entries j < min(floor((t+1)/r), nc) } (idx == NULL, HCA)
 *  union { raw positions s, max(0, t-W+1) <= s <= t } read from slot s mod ring
 * of kw / vw, under ONE softmax of scale * q . key:
 *   o[b, i, h] = sum p v,  lse[b, i, h] = natural log of the softmax denominator.
 *   q [batch, T, H, D]   kc, vc [batch, nc_cap, D]   idx [batch, T, k] or NULL
 *   kw, vw [batch, ring, D] (prefill: the raw K/V with ring = L; decode: a
 *   ring of at least W slots)   o [batch, T, H, D]   lse [batch, T, H] fp32 or NULL
 * `mode` picks the schedule (HYB_ATTN_DECODE splits each query's keys over
 * several CTAs and merges the partial softmaxes); both compute the same
 * function.  Entries of idx outside [0, V) other than -1 are skipped and
 * reported as HYB_ERR_DEVICE_CHECK.  Scratch: `ws` of at least
 * hyb_attn_fwd_workspace_size(...) bytes (may be 0 for PREFILL).
 * mode | HYB_ATTN_REAL_KV (CSA with idx only; bf16, H = 64, D = 128): the "real
 * K/V" reading -- each selected entry j stands for its raw tokens jr .. jr+r-1,
 * read from the ring, and the key set is those tokens and the window as a set
 * of raw positions (a token the window holds is not repeated).  kc / vc are not
 * read (may be NULL); the ring must still hold every selected token (in decode a
 * full raw K/V cache with ring > t); a token that has left the ring is reported
 * as HYB_ERR_DEVICE_CHECK.
 */
size_t hyb_attn_fwd_workspace_size(int dtype, int batch, int T, int H, int D, int k,
                                   int nc, int W, int mode);
int hyb_attn_fwd(int dtype, int batch, int T, int H, int D,
                 const void* q, const int* q_pos,
                 const void* kc, const void* vc, int nc, int nc_cap, int r,
                 const int* idx, int k,
                 const void* kw, const void* vw, int ring, int W, float scale,
                 void* o, float* lse, int mode,
                 void* ws, size_t ws_bytes, hyb_stream_t stream);

/*
 * Test hook for the bounded device waits (no counterpart on the pages: it
 * exists to exercise the failure path).  Same arguments and results as
 * hyb_attn_fwd for the tensor-core path it covers (bf16, H = 64, D = 128, not
 * the real-K/V reading), plus:
 *  - wait_ns (1 .. 1e9): the limit of every wait inside the attention kernel
 *    instead of 1 s;
 *  - drop_arrival != 0: the first CTA withholds one arrival on its first K
 *    tile, so that its waits expire; that CTA then stops, lets the MMAs it
 *    issued finish, frees its tensor memory and records HYB_ERR_TIMEOUT in the
 *    status word (read with hyb_get_device_status).  The outputs of the queries
 *    that CTA owned are left unspecified; the device and the stream stay usable.
 * Returns HYB_ERR_INVALID_ARG for wait_ns outside 1 .. 1e9 and
 * HYB_ERR_UNSUPPORTED for shapes the hook does not cover.
 */
int hyb_attn_fwd_wait_test(int dtype, int batch, int T, int H, int D,
                           const void* q, const int* q_pos,
                           const void* kc, const void* vc, int nc, int nc_cap, int r,
                           const int* idx, int k,
                           const void* kw, const void* vw, int ring, int W, float scale,
                           void* o, float* lse, int mode,
                           void* ws, size_t ws_bytes, hyb_stream_t stream,
                           unsigned long long wait_ns, int drop_arrival);

#ifdef __cplusplus
}
#endif

#endif /* HYB_H_ */
