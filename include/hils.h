/*
 * hils.h -- C ABI of HiLS (Hierarchical Landmark Sparse) attention on NVIDIA
 * B200 (sm_100a): the forward (prefill and decode), its backward with the
 * chunk selection held fixed, and the decode step split over several GPUs.
 *
 * The method ("Hierarchical Sparse Attention Done Right"; ai-feeds.com digest,
 * section 方法; oopus.info review, section 二; chatpaper abstract):
 *   a1  low-rank query calibration      q~ = q + (q A) B            (digest, 输入与分块)
 *   a2  landmark scoring                s_j = q~ . lm_j / sqrt(d)   (digest, 关键模块 item 1)
 *   a3  selection: own chunk c(i) = floor(i/S) plus the top-(k-1) chunks j < c(i),
 *       ordered by (score desc, chunk index asc)                    (digest, 关键模块 item 2)
 *   a4  fusion weights w = softmax(selected scores)                 (digest, item 1 outer softmax)
 *   a5  per-chunk attention O_j = softmax(q K_j^T / sqrt(d)) V_j with the raw q,
 *       keys at positions <= i in the own chunk                     (abstract; digest item 2)
 *   a6  fused output out = sum_j w_j O_j                            (review, 融合; abstract)
 *   a7  chunk-granular paged KV access: one page = one chunk        (digest, 关键模块 item 3)
 *   a8  decode step: append k_t, v_t, then row t of the prefill     (digest, 局限: per-step scan)
 *   backward of a1..a6 with the selection fixed                      (digest, 关键模块 items 1, 3;
 *                                                                     输出与训练)
 *
 * Conventions shared by every entry point:
 *   - All tensor arguments are caller-owned DEVICE pointers, 16-byte aligned,
 *     densely packed in the layouts below (row-major, last index fastest).
 *     The library allocates nothing; scratch comes from the caller's workspace.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Every call is
 *     asynchronous on that stream; none synchronises the device.
 *   - Arguments are validated on the host before anything is launched; a bad
 *     argument returns an error status and launches nothing.  The message of the
 *     last failure on the calling thread is available from hils_last_error().
 *   - Kernels check block-table entries against num_pages and chunk indices
 *     against max_chunks; an out-of-range entry skips the access and sets a
 *     device error word that hils_device_status() reports and clears.
 *   - Inputs are assumed finite.
 *   - Shapes: head_dim 64 or 128; chunk_size 64; 1 <= top_k <= 32;
 *     0 <= calib_rank <= 64; n_q_heads a multiple of n_kv_heads.
 */
#ifndef HILS_H_
#define HILS_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  HILS_OK = 0,
  HILS_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misaligned pointer */
  HILS_ERR_UNSUPPORTED = 2,   /* valid but not implemented (e.g. head_dim 96) */
  HILS_ERR_WORKSPACE = 3,     /* workspace smaller than hils_workspace_size() */
  HILS_ERR_CUDA = 4,          /* a CUDA launch or runtime call failed */
  HILS_ERR_TIMEOUT = 5,       /* a bounded device-side wait ran out */
  HILS_ERR_DEVICE_CHECK = 6   /* a device-side bounds check fired */
} hils_status;

typedef enum { HILS_F32 = 0, HILS_BF16 = 1 } hils_dtype;

typedef enum {
  HILS_OP_SCORE = 0,
  HILS_OP_TOPK = 1,
  HILS_OP_PREFILL = 2,
  HILS_OP_DECODE = 3,
  HILS_OP_PREFILL_BACKWARD = 4
} hils_op;

typedef struct {
  int32_t batch;       /* B: sequences */
  int32_t n_q_heads;   /* Hq */
  int32_t n_kv_heads;  /* Hkv; query head h reads KV head h / (Hq/Hkv) */
  int32_t head_dim;    /* d: 64 or 128 */
  int32_t chunk_size;  /* S: 64 (one chunk = one KV page) */
  int32_t top_k;       /* k: own chunk + (k-1) retrieved chunks, 1..32 */
  int32_t calib_rank;  /* r: rank of the calibration A [d][r], B [r][d]; 0 = none */
  int32_t dtype;       /* hils_dtype of q, K, V, landmarks, k_new, v_new and out */
} hils_config;

/* Paged, chunk-granular KV cache (all device memory, owned by the caller). */
typedef struct {
  void* pages;                /* [num_pages][2][n_kv_heads][chunk_size][head_dim], [.][0] = K, [.][1] = V */
  int64_t num_pages;
  const int32_t* block_table; /* [batch][max_chunks]: logical chunk j of sequence b -> page */
  int32_t max_chunks;
  const void* landmarks;      /* [batch][max_chunks][n_kv_heads][head_dim]: one landmark key per chunk
                                 and KV head, supplied by the caller for every chunk in use,
                                 including a partially filled last chunk */
  int32_t* seq_lens;          /* [batch] tokens present; read by hils_decode, advanced by it when appending */
} hils_kv_cache;

/* Bytes of workspace that `op` needs for this configuration.  q_len is the
 * number of query positions per sequence (prefill; 1 for decode) and
 * max_chunks the cache's block-table width.  Returns 0 when none is needed or
 * on a bad argument (then hils_last_error() says which). */
size_t hils_workspace_size(const hils_config* cfg, int op, int64_t q_len, int32_t max_chunks);

/* a1 + a2 materialised, for tests and small inputs.
 * q       [B][q_len][Hq][d]  queries at positions q_pos0 .. q_pos0+q_len-1
 * A, B    float32 [d][r], [r][d], 16-byte aligned (ignored when calib_rank == 0)
 * scores  float32 [B][q_len][Hq][n_cols]; column j holds s_j for j <= floor(pos/S)
 *         and -inf after it.  Requires floor((q_pos0+q_len-1)/S) < n_cols <= max_chunks. */
int hils_score(const hils_config* cfg, const void* q, int64_t q_len, int64_t q_pos0, const float* A,
               const float* B, const hils_kv_cache* cache, float* scores, int32_t n_cols,
               void* stream);

/* a3 + a4 on materialised scores (layout as hils_score writes it).
 * idx  int32 [B][q_len][Hq][k]: slot 0 = own chunk, then the selected chunks by
 *      (score desc, index asc); -1 pads when fewer than k chunks are visible.
 * w    float32, same shape: softmax of the selected scores, 0 in padded slots. */
int hils_topk(const hils_config* cfg, const float* scores, int64_t q_len, int64_t q_pos0,
              int32_t n_cols, int32_t* idx, float* w, void* stream);

/* a1..a7: the full prefill forward, without materialising scores.
 * q       [B][q_len][Hq][d] at positions q_pos0 .. q_pos0+q_len-1 of every sequence;
 *         the cache must hold tokens 0 .. q_pos0+q_len-1 (seq_lens is not read).
 * out     [B][q_len][Hq][d] in cfg->dtype.
 * idx_out, w_out  optional [B][q_len][Hq][k] copies of the selection (may be NULL).
 * ws      workspace of at least hils_workspace_size(cfg, HILS_OP_PREFILL, q_len, max_chunks) bytes,
 *         256-byte aligned; its contents need not be initialised. */
int hils_prefill(const hils_config* cfg, const void* q, int64_t q_len, int64_t q_pos0,
                 const float* A, const float* B, const hils_kv_cache* cache, void* out,
                 int32_t* idx_out, float* w_out, void* ws, size_t ws_bytes, void* stream);

/* Backward of hils_prefill with the chunk selection held fixed: the gradients
 * of sum(dout * out) for training end to end under the language-modelling
 * loss (the digest, 关键模块 item 1: the retrieval scores are differentiable
 * and optimised by that loss, item 3: native sparse training; 输出与训练).
 * The selection is a discrete choice and has no gradient; the fusion weights
 * (through the landmark scores and the calibration), the per-chunk attention
 * and the calibration do.  Per row, with the forward's notation:
 *   dw_j = dout . O_j,  ds_j = w_j (dw_j - sum_l w_l dw_l),
 *   dq~ = sum_j ds_j lm_j / sqrt(d),  dlm_j += ds_j q~ / sqrt(d),
 *   per chunk with G = w_j dout: dV += P_j^T G, dS = P_j (G V_j^T - G . O_j),
 *     dq += dS K_j / sqrt(d), dK += dS^T q / sqrt(d),
 *   dq += dq~ + (dq~ B^T) A^T,  dA += q^T (dq~ B^T),  dB += (qA)^T dq~.
 * q, q_len, q_pos0, A, B, cache  as given to hils_prefill (seq_lens not read).
 * idx, w     int32 / float32 [B][q_len][Hq][k]: the forward's selection and
 *            weights (hils_prefill's idx_out and w_out).
 * out        [B][q_len][Hq][d] in cfg->dtype, 16-byte aligned: the forward's
 *            output for the same inputs.  sum_l w_l dw_l = dout . out, so the
 *            bf16 head_dim-128 path takes that row term from it before the
 *            attention pass; the other configurations sum the dw_l instead.
 * dout       [B][q_len][Hq][d] in cfg->dtype, 16-byte aligned.
 * dq         float32 [B][q_len][Hq][d], 16-byte aligned.
 * dpages     float32 [num_pages][2][Hkv][S][d], the gradient of the page pool
 *            (same layout as cache->pages).
 * dlandmarks float32 [B][max_chunks][Hkv][d].
 * dA, dB     float32 [d][r], [r][d] (may be NULL when calib_rank == 0).
 * All five gradients are ADDED INTO: zero them before the first call; a long
 * prefill split into query blocks (q_pos0 > 0) then accumulates its blocks'
 * gradients of the shared pages, landmarks, A and B.  The order of the float
 * additions is not fixed, so results may differ in the last bits from run
 * to run.  Arithmetic is float32, except that for bf16 storage at head_dim
 * 128 the per-chunk attention products run on the tensor cores with bf16
 * operands (the probabilities, G = w dout, dS and ds rounded to bf16, as the
 * forward rounds the probabilities) and float32 accumulation.
 * ws         at least hils_workspace_size(cfg, HILS_OP_PREFILL_BACKWARD, q_len,
 *            max_chunks) bytes, 256-byte aligned; its contents need not be
 *            initialised.
 * Errors: HILS_ERR_INVALID_ARG (a missing or misaligned pointer, a query
 * position beyond the block table), HILS_ERR_UNSUPPORTED (configuration),
 * HILS_ERR_WORKSPACE (ws too small); nothing is queued when a check fails.
 * A block-table entry or selected chunk out of range is reported by
 * hils_device_status(). */
int hils_prefill_backward(const hils_config* cfg, const void* q, int64_t q_len, int64_t q_pos0,
                          const float* A, const float* B, const hils_kv_cache* cache,
                          const int32_t* idx, const float* w, const void* out,
                          const void* dout, float* dq, float* dpages, float* dlandmarks,
                          float* dA, float* dB, void* ws, size_t ws_bytes, void* stream);

/* a8: one decode step for every sequence of the batch.
 * q             [B][Hq][d]: one query per sequence.
 * k_new, v_new  [B][Hkv][d], 16-byte aligned, or both NULL.  When given, each
 *               sequence's new token is written at position t = seq_lens[b] (its
 *               chunk's page must be in the block table) and seq_lens[b] is advanced
 *               to t+1 on the device at the end of the step, so repeated calls (or a
 *               captured graph) walk forward.
 *               When NULL, the token at t = seq_lens[b]-1 must already be present.
 * out           [B][Hq][d] in cfg->dtype; idx_out, w_out optional [B][Hq][k].
 * ws            at least hils_workspace_size(cfg, HILS_OP_DECODE, 1, max_chunks) bytes,
 *               256-byte aligned; zero it once before the first call (cudaMemset)
 *               and keep it for later calls with the same configuration: its
 *               completion counters return to zero at the end of every step. */
int hils_decode(const hils_config* cfg, const void* q, const void* k_new, const void* v_new,
                const float* A, const float* B, hils_kv_cache* cache, void* out, int32_t* idx_out,
                float* w_out, void* ws, size_t ws_bytes, void* stream);

/* Context-parallel decode: one sequence's chunks spread over several GPUs
 * (the decode step beyond one GPU's memory).  Each GPU ("rank") holds the
 * chunks chunk_base .. chunk_base + shard->max_chunks - 1 of every sequence:
 * `shard` is a cache of its own (pages, block table and landmarks indexed by
 * local chunk, j - chunk_base), and shard->seq_lens holds the global token
 * counts, the same on every rank.  t = seq_lens[b] when appending (k_new and
 * v_new given), else seq_lens[b] - 1; the own chunk is t / chunk_size.  One
 * step is four calls around two collectives that the caller runs (NCCL, for
 * instance); the pieces follow the paper's fusion (review, 二: each chunk's
 * attention weighted by its retrieval score; digest, 局限: every landmark is
 * scored at every step), split so that only the candidate lists and the
 * d-vectors of the weighted outputs cross between GPUs:
 *   1. hils_decode_cp_candidates: this shard's best k-1 chunks before the
 *      own one, per (sequence, query head), as 64-bit selection keys, best
 *      first, into keys [B][Hq][k-1] (key 0 = none; a larger key ranks higher
 *      in (score desc, chunk asc): the high word is the float32 score mapped
 *      to an unsigned order, the low word is the complement of the global
 *      chunk index), and the own chunk's score into own_score [B][Hq] on the
 *      rank holding it (-inf elsewhere).  That rank appends k_new, v_new.
 *      ws: the shard's decode workspace, at least hils_workspace_size(cfg,
 *      HILS_OP_DECODE, 1, shard->max_chunks) bytes, 256-byte aligned, zeroed
 *      once before the first call and kept (as for hils_decode).
 *   2. all-gather of keys and own_score over the ranks, in rank order.
 *   3. hils_decode_cp_select: the global selection and fusion weights from
 *      the gathered keys [world][B][Hq][k-1] and own scores [world][B][Hq],
 *      into idx and w [B][Hq][k] (global chunk indices; the same on every
 *      rank, and the same slot order and weights as hils_decode).
 *   4. hils_decode_cp_attend: the weighted outputs of the selected chunks
 *      this shard holds, float32 partial [B][Hq][d] (zero where none).
 *   5. all-reduce (sum) of partial.
 *   6. hils_decode_cp_finish: out [B][Hq][d] in cfg->dtype from the sum;
 *      seq_lens advanced by one when `append` (call it on every rank, each
 *      with its own seq_lens).
 * All arrays are device memory; nothing is allocated.  Steps 1 and 4 run
 * the kernels of hils_decode (the chunk ranges of the scan spread over CTAs,
 * the selected chunks over a cluster of CTAs per head) on the shard.  A step's calls go to
 * one stream per rank, in this order.  The own chunk must be held by exactly
 * one rank; hils_device_status() reports HILS_ERR_DEVICE_CHECK otherwise. */
int hils_decode_cp_candidates(const hils_config* cfg, const void* q, const void* k_new,
                              const void* v_new, const float* A, const float* B,
                              hils_kv_cache* shard, int64_t chunk_base, uint64_t* keys,
                              float* own_score, void* ws, size_t ws_bytes, void* stream);
int hils_decode_cp_select(const hils_config* cfg, int32_t world, const uint64_t* keys,
                          const float* own_scores, const int32_t* seq_lens, int32_t append,
                          int32_t* idx, float* w, void* stream);
int hils_decode_cp_attend(const hils_config* cfg, const void* q, const void* k_new,
                          const void* v_new, const hils_kv_cache* shard, int64_t chunk_base,
                          const int32_t* idx, const float* w, float* partial, void* stream);
int hils_decode_cp_finish(const hils_config* cfg, const float* sum, void* out, int32_t* seq_lens,
                          int32_t append, void* stream);

/* The decode step without a workspace argument, for callers that cannot
 * allocate device memory: plugins run by a host engine that owns every device
 * allocation and passes kernels only their inputs and outputs, and services
 * that must not allocate once they are serving (cudaMalloc can synchronise the
 * device and can fail under memory pressure).  The paper has no counterpart:
 * this is a deployment convenience around hils_decode.
 * Arguments and results are those of hils_decode.  Its scratch is one array of
 * hils_decode_noalloc_capacity() bytes (4 MiB) built into the library, which
 * every GPU that loads the library holds until the process exits; a
 * configuration that needs more returns HILS_ERR_WORKSPACE (use hils_decode).
 * The first call on each device looks up the array's device address; make
 * that first call before any stream capture, and make no call after
 * cudaDeviceReset (the looked-up address is kept for the life of the
 * process).  Each call that passes its argument checks clears the array's
 * completion counters (a cudaMemsetAsync on `stream`) and otherwise reuses
 * what the previous call left there; a rejected call queues nothing.  All
 * calls on one device share the array: calls that overlap on the GPU (other
 * streams, other threads) race and give wrong results, so serialise them.
 * Allocates no memory. */
int hils_decode_noalloc(const hils_config* cfg, const void* q, const void* k_new,
                        const void* v_new, const float* A, const float* B, hils_kv_cache* cache,
                        void* out, int32_t* idx_out, float* w_out, void* stream);
size_t hils_decode_noalloc_capacity(void);

/* Synchronises `stream`, then reports and clears the device error word set by
 * the kernels' checks: HILS_OK; HILS_ERR_TIMEOUT if a kernel gave up on a bounded
 * wait (the results of that call are undefined; later calls are unaffected);
 * HILS_ERR_DEVICE_CHECK if only a bounds check fired (HILS_ERR_CUDA if the
 * synchronisation itself failed). */
int hils_device_status(void* stream);

/* Testing hook for the failure path: every kernel wait on another stage of its
 * pipeline gives up after `ns` nanoseconds (0 restores the default, 2 s), after
 * which the kernel lets its own asynchronous copies and products finish, exits
 * and reports HILS_ERR_TIMEOUT through hils_device_status().  A short limit
 * makes calls give up while their pipelines are still filling.  Applies to the
 * current device; not meant for production use. */
int hils_set_wait_limit_ns(uint64_t ns);

/* Kernel timing with CUDA events, for benchmarking (not thread-safe).
 * hils_profile_enable(1): from now on every kernel the library launches is
 * bracketed by an event pair recorded on the call's stream.
 * hils_profile_collect(): waits for the recorded events and adds their
 * elapsed times to per-phase totals (phase = kernel name, e.g. "prefill.select").
 * hils_profile_read(i, ...): phase i's name, total milliseconds and launch
 * count; returns HILS_ERR_INVALID_ARG past the last phase.
 * hils_profile_reset(): collects pending events, then clears the totals. */
int hils_profile_enable(int on);
int hils_profile_collect(void);
int hils_profile_read(int i, const char** name, double* total_ms, long long* launches);
int hils_profile_reset(void);

/* Message of the last failed call on this thread ("" if none). */
const char* hils_last_error(void);

/* Library version, e.g. "hils-b200 0.1.0 sm_100a". */
const char* hils_version(void);

#ifdef __cplusplus
}
#endif

#endif /* HILS_H_ */
