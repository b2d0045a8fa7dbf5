/*
 * msa.h — C ABI of the B200 (sm_100a) library for the hot path of MiniMax Sparse
 * Attention (MSA).
 *
 * What the library computes (hyper.ai "MiniMax Sparse Attention", Method; zhichai.net
 * article, section 2 "Index Branch" / "Main Branch"):
 *   Index Branch, per GQA group g and query i:
 *     s_g(i, j) = q_idx[i, g] . k_idx[j, g] for every causally visible token j <= i;
 *     S_g(i, b) = max of s_g(i, j) over the tokens j <= i of block b (Block Max
 *     Pooling, blocks of Bk = 128 tokens);
 *     block_ids[i, g, :] = the local block b_l = floor(i / Bk) plus the k - 1 best other
 *     visible blocks by S (higher first, lower block index first among equal scores);
 *     when b_l + 1 <= k every visible block is taken. Rows list ids in ascending
 *     order and are padded with -1.
 *   Main Branch, per query head h of group g = h / (Hq / G):
 *     o[i, h] = softmax(q[i, h] . k[j, g] * scale) . v[j, g] over the tokens j <= i of
 *     the selected blocks (scale 1/sqrt(d) unless given).
 *   Decode applies the same definition to one new query per sequence, at position
 *   seqlens[b] - 1 of that sequence's cache.
 *
 * Conventions for every entry point:
 *   - Tensors are row-major and contiguous, bf16 passed as raw 16-bit storage
 *     (const void*). Every pointer is a DEVICE pointer owned by the caller, 16-byte
 *     aligned, except the input and output buffers of msa_forward_host, which are host
 *     memory. The library allocates and frees no memory; scratch memory comes from the
 *     caller's workspace (size from the matching *_workspace function; 256-byte
 *     aligned base). It keeps up to three extra streams per device of its own (see
 *     msa_forward_host) and creates its events per call.
 *   - stream is a cudaStream_t (NULL = legacy default stream). All work is enqueued on
 *     it; no call synchronises the host, except msa_get_device_error.
 *   - Arguments are validated before anything is enqueued. A bad argument returns
 *     MSA_ERR_INVALID_ARG, a valid but unimplemented shape MSA_ERR_UNSUPPORTED, a too
 *     small workspace MSA_ERR_WORKSPACE, a failed CUDA launch MSA_ERR_CUDA; nothing is
 *     launched in those cases. msa_last_error_detail() then describes the failure.
 *   - Faults detected on the device (a pipeline wait that timed out, an index out of
 *     range) are recorded in a per-device error word and reported by
 *     msa_get_device_error(); the kernel that saw it returns early, so the output of
 *     that call is undefined.
 *   - Supported shapes: Bk in {32, 64, 128} (the block sizes of the hyper.ai page's
 *     block-size ablation, Experiment); d in {64, 128}; d_idx in {32, 64, 128};
 *     R = Hq / G in {1, 2, 4, 8, 16}; 1 <= k <= 32 (Bk < 128: k in {4, 8, 16, 32});
 *     1 <= N < 2^26, within the per-entry sequence limits stated below (checked before
 *     anything is enqueued).
 */
#ifndef MSA_H_
#define MSA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MSA_API __attribute__((visibility("default")))
#else
#define MSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum msa_status_t {
  MSA_OK = 0,
  MSA_ERR_INVALID_ARG = 1,
  MSA_ERR_UNSUPPORTED = 2,
  MSA_ERR_WORKSPACE = 3,
  MSA_ERR_CUDA = 4,
  MSA_ERR_TIMEOUT = 5,
  MSA_ERR_DEVICE_BOUNDS = 6
} msa_status_t;

typedef enum msa_mode_t { MSA_MODE_PREFILL = 0, MSA_MODE_DECODE = 1 } msa_mode_t;

/* Shapes of one msa_forward call.
 *   prefill: n = N tokens of one sequence; q [N, hq, d]; k, v [N, g, d];
 *            q_idx, k_idx [N, g, d_idx]; o [N, hq, d]; block_ids [N, g, k].
 *   decode:  n = B sequences, one new query each; q [B, hq, d]; q_idx [B, g, d_idx];
 *            caches k, v [B, lmax, g, d] and k_idx [B, lmax, g, d_idx], where the new
 *            token's k / v / k_idx are already stored at position seqlens[b] - 1;
 *            seqlens: device int32 [B], 1 <= seqlens[b] <= lmax; o [B, hq, d];
 *            block_ids [B, g, k].
 * query_chunk (prefill): queries per attention chunk, a multiple of 128; 0 picks the
 * library default. Larger chunks use more workspace; it is raised where needed so that a
 * sequence has at most 128 chunks (the results do not depend on it).
 * lse_out (prefill, msa_forward only; NULL to skip): device float [N, hq], the natural-log
 * log-sum-exp of each (query, head)'s scaled logits over its selected tokens, as
 * msa_index_kl takes it. */
typedef struct msa_params {
  int32_t mode;
  int32_t hq, g, d, d_idx, bk, k;
  float scale;               /* 0 => 1 / sqrt(d) */
  int64_t n;
  int64_t lmax;              /* decode only */
  const int32_t* seqlens;    /* decode only, device pointer */
  int64_t query_chunk;       /* prefill only */
  float* lse_out;            /* prefill only, msa_forward only, nullable */
} msa_params;

/* Index Branch (scores, Block Max Pooling, Top-k with the local block forced).
 * Defined by hyper.ai "MiniMax Sparse Attention", Method (second paragraph: per GQA group a
 * dot-product score of every visible key token, Block Max Pooling, the Top-K blocks with the
 * local block always included) and zhichai.net section 2 "Index Branch" (one index query head
 * and one shared index key head per group); the selection is exp-free (zhichai.net section
 * 4.1: only the order of the scores matters).
 * q_idx, k_idx: [n, g, d_idx] bf16. block_ids (out): [n, g, k] int32, caller-owned.
 * Workspace: msa_index_select_workspace(...) bytes (a few hundred bytes when the one-kernel
 * path serves (n, k); the block maxima otherwise). Paths: the one-kernel path (Top-k in the
 * score epilogue, no block maxima in memory) serves k in {4, 8, 16, 32} at every length and
 * every Bk; any other k takes the two-kernel path (Bk = 128 only), which serves at most 32768
 * query blocks (4,194,304 tokens); longer sequences return MSA_ERR_UNSUPPORTED and the
 * workspace query returns 0.
 * Returns MSA_OK or an error as described above. */
MSA_API size_t msa_index_select_workspace(int64_t n, int32_t g, int32_t d_idx, int32_t bk, int32_t k);
MSA_API msa_status_t msa_index_select(const void* q_idx, const void* k_idx, int64_t n, int32_t g, int32_t d_idx,
                              int32_t bk, int32_t k, int32_t* block_ids, void* workspace,
                              size_t workspace_bytes, void* stream);

/* Index Branch for callers that cannot allocate device memory. This entry point has no
 * counterpart in the method's description; it exists for callers that only hold a stream
 * and raw tensor pointers, such as a plugin running inside another framework's execution
 * engine or a serving loop that forbids device allocations after start-up, and so cannot
 * call cudaMalloc to provide the workspace msa_index_select needs. It computes exactly what
 * msa_index_select computes, with the same arguments minus the workspace.
 *   Scratch: when the one-kernel path serves (n, k) (see msa_index_select) no scratch is
 *   needed at all. Otherwise the two-kernel path keeps the block maxima in a 32 MiB array
 *   inside the library's device image. Every GPU that loads the library holds that array until
 *   the process exits. The query blocks are processed in as many launches as it takes for each
 *   launch's maxima to fit; a problem whose single last query block needs more than 32 MiB
 *   (4 * g * 128 * (ceil(n/128) - 1) bytes), or that exceeds the two-kernel path's sequence
 *   limit, is rejected with MSA_ERR_UNSUPPORTED before anything is enqueued.
 *   Nothing is allocated: no cudaMalloc, cudaFree or allocating library routine is called.
 *   The scratch needs no zeroing (every entry is written before it is read).
 *   Set-up: the first call on a device looks up the array's device address (once per device,
 *   with that device current); make that first call before any stream capture.
 *   Calls on one device share the scratch: calls that overlap on the GPU (different streams,
 *   or different host threads without ordering) race and give undefined results. */
MSA_API msa_status_t msa_index_select_static(const void* q_idx, const void* k_idx, int64_t n, int32_t g,
                                             int32_t d_idx, int32_t bk, int32_t k, int32_t* block_ids,
                                             void* stream);

/* Main Branch given the selection, executed KV-outer (each K/V block is held on chip
 * while the queries that chose it stream through; per-slot partial results are
 * merged by a deterministic log-sum-exp pass, no atomics).
 * Defined by hyper.ai "MiniMax Sparse Attention", Method (third paragraph: standard scaled
 * dot-product softmax attention restricted to the tokens of the selected blocks) and
 * zhichai.net section 2 "Main Branch" (every query head of a group shares the group's block
 * set); the KV-outer execution without atomic updates follows the same page's Key
 * Contributions and zhichai.net section 4.2.
 * q: [n, hq, d]; k, v: [n, g, d]; block_ids: [n, g, topk] as produced by
 * msa_index_select (ascending, -1 padded, each id <= floor(i / bk)); o (out):
 * [n, hq, d] bf16, caller-owned. scale 0 => 1 / sqrt(d). Sequence limit: at most 14528
 * blocks (1,859,584 tokens at Bk = 128; the inverted index keeps one 128-bit mask per block
 * on chip).
 * Ids that break the rules above are reported through msa_get_device_error as
 * MSA_ERR_DEVICE_BOUNDS and their rows skipped. */
MSA_API size_t msa_sparse_attn_workspace(int64_t n, int32_t hq, int32_t g, int32_t d, int32_t bk, int32_t topk);
MSA_API msa_status_t msa_sparse_attn(const void* q, const void* k, const void* v, const int32_t* block_ids, int64_t n,
                             int32_t hq, int32_t g, int32_t d, int32_t bk, int32_t topk, float scale, void* o,
                             void* workspace, size_t workspace_bytes, void* stream);

/* Both branches in one call: prefill (Index Branch then KV-outer Main Branch) or
 * decode (query-stationary index scan, Top-k, sparse attention over the selected
 * blocks, merge). block_ids_out may be NULL (the selection then lives in the
 * workspace).
 * Prefill computes msa_index_select followed by msa_sparse_attn (hyper.ai page, Method,
 * second and third paragraphs) and takes the stricter of their sequence limits. Decode applies
 * the same definition to the last token of each sequence: one query per sequence cannot fill
 * a KV-stationary tile, so it runs query-stationary, the design the skandtandon.pages.dev note
 * "KV-stationary attention" (The problem) contrasts with the KV-stationary one.
 * The call only enqueues kernel launches on `stream` (no host synchronisation, no
 * allocation) with grids that depend on *p alone (decode: on lmax; the lengths are read on
 * the device), so it may be captured into a CUDA graph and the graph replayed on new
 * contents of the same buffers. */
MSA_API size_t msa_forward_workspace(const msa_params* p);
MSA_API msa_status_t msa_forward(const msa_params* p, const void* q, const void* k, const void* v, const void* q_idx,
                         const void* k_idx, int32_t* block_ids_out, void* o, void* workspace,
                         size_t workspace_bytes, void* stream);

/* Index-branch KL loss, forward: per (query i, group g), KL(P_main || P_idx) over the tokens
 * T of the selected blocks (j <= i), in natural-log units. Defined by hyper.ai "MiniMax Sparse
 * Attention", Method (fourth paragraph: a KL divergence aligns the Index Branch's probability
 * distribution with the Main Branch's on the selected tokens) and zhichai.net section 5.1 (the
 * Main Branch side is the group-averaged distribution). The pages leave the index distribution
 * open; this library takes P_main(j) = mean over the group's heads h of
 * exp(scale q[i,h].k[j,g] - lse[i,h]) and P_idx = softmax over T of idx_scale * q_idx[i,g].k_idx[j,g]
 * (idx_scale 0 => 1 / sqrt(d_idx)).
 * p: prefill shapes (mode MSA_MODE_PREFILL; lse_out ignored), hq / g <= 8. q [n, hq, d],
 * k [n, g, d], q_idx / k_idx [n, g, d_idx] bf16; block_ids [n, g, k] and lse [n, hq] float as
 * msa_forward produced them (lse via msa_params.lse_out); kl (out): device float [n, g].
 * Executed KV-outer like the Main Branch: per (query, selected block) partial sums, merged per
 * query in ascending slot order (deterministic, no atomics). Workspace:
 * msa_index_kl_workspace(p) bytes (0 = unsupported shape). Sequence limit: as msa_sparse_attn. */
MSA_API size_t msa_index_kl_workspace(const msa_params* p);
MSA_API msa_status_t msa_index_kl(const msa_params* p, const void* q, const void* k, const void* q_idx,
                                  const void* k_idx, const int32_t* block_ids, const float* lse, float idx_scale,
                                  float* kl, void* workspace, size_t workspace_bytes, void* stream);

/* Prefill with the inputs and the output in HOST memory (no counterpart in the method's
 * description: it computes msa_forward's prefill and adds the copies). q, k, v, q_idx, k_idx and o are
 * host pointers with the shapes of msa_forward's prefill (block_ids_out: host [n, g, k] or
 * NULL); page-locked memory lets the copies overlap the kernels (pageable memory works, the
 * copies then serialise with the host). device_buf (device, 256-byte aligned,
 * msa_forward_host_device_bytes(p) bytes) receives device copies of the inputs and of o,
 * and the msa_forward workspace. Within the call the index inputs are copied first, the
 * Index Branch starts as soon as they land while q / k / v are copied behind it chunk by
 * chunk (query_chunk rows) on a second stream; each chunk's Main Branch starts once its rows
 * are resident, and its output rows are copied back on a third stream while later chunks
 * compute. Everything is ordered after earlier work on `stream`, and the host output (and
 * block ids) are complete once `stream` is. Prefill only (decode returns
 * MSA_ERR_UNSUPPORTED). Calls that share `stream` may reuse one device_buf. */
MSA_API size_t msa_forward_host_device_bytes(const msa_params* p);
MSA_API msa_status_t msa_forward_host(const msa_params* p, const void* q, const void* k, const void* v,
                                      const void* q_idx, const void* k_idx, int32_t* block_ids_out, void* o,
                                      void* device_buf, size_t device_bytes, void* stream);

/* Failure reporting of this library (no counterpart in the method's description).
 * Synchronises `stream`, then reads and clears this device's error word. Returns
 * MSA_OK, MSA_ERR_TIMEOUT or MSA_ERR_DEVICE_BOUNDS (the first error recorded since the
 * last call), or MSA_ERR_CUDA when the synchronisation itself failed. */
MSA_API msa_status_t msa_get_device_error(void* stream);

/* Failure detection (no counterpart in the method's description). Every pipeline wait of the
 * library's kernels is bounded: a wait that gates new work gives up after this limit (default
 * and maximum 2 s; ns = 0 restores the default), records MSA_ERR_TIMEOUT for
 * msa_get_device_error and makes the kernel stop issuing work; waits for work already in
 * flight (loads, products, stores) always use the 2 s default, so the kernel drains it before
 * it returns and the context stays usable. A short limit makes every such call fail with
 * MSA_ERR_TIMEOUT (a way to exercise that path); its outputs are then undefined. The limit
 * is per device (the current one) and applies to kernels launched after the call returns. */
MSA_API msa_status_t msa_set_wait_limit_ns(uint64_t ns);

/* Per-kernel timing (instrumentation for benchmarks, no counterpart in the method's
 * description; off by default).
 * msa_profile_start() makes every later launch by this library, on any stream, record a
 * CUDA event before and after itself. msa_profile_stop() waits for those events, stops
 * recording and fills out[0 .. min(count, max_out)) with one entry per kernel kind that
 * ran (name, launches, summed device milliseconds); it returns count, or -1 on a CUDA
 * error. */
typedef struct msa_kernel_stat {
  const char* name;
  int32_t launches;
  double total_ms;
} msa_kernel_stat;
MSA_API msa_status_t msa_profile_start(void);
MSA_API int32_t msa_profile_stop(msa_kernel_stat* out, int32_t max_out);

/* Static English name of a status code. */
MSA_API const char* msa_status_string(msa_status_t status);

/* Text of the last validation or launch failure seen by this host thread ("" if none). */
MSA_API const char* msa_last_error_detail(void);

#ifdef __cplusplus
}
#endif

#endif /* MSA_H_ */
