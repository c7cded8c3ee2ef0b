// C-ABI entry points of the HiLS library (declared in include/hils.h):
// argument validation on the host, workspace carve-up, kernel dispatch.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>

#include <map>
#include <mutex>
#include <utility>

#include "hils_common.cuh"

namespace {

thread_local std::string g_last_error;

int fail(int status, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return status;
}

int cuda_fail(cudaError_t e, const char* where) {
  return fail(HILS_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

// Checks shared by every entry point; fills the kernel parameters.
int check_config(const hils_config* c, hils::Params* P) {
  if (!c) return fail(HILS_ERR_INVALID_ARG, "config is NULL");
  if (c->batch < 0 || c->n_q_heads <= 0 || c->n_kv_heads <= 0)
    return fail(HILS_ERR_INVALID_ARG, "batch, n_q_heads, n_kv_heads must be positive");
  if (c->n_q_heads % c->n_kv_heads != 0)
    return fail(HILS_ERR_INVALID_ARG, "n_q_heads (%d) is not a multiple of n_kv_heads (%d)",
                c->n_q_heads, c->n_kv_heads);
  if (c->head_dim != 64 && c->head_dim != 128)
    return fail(HILS_ERR_UNSUPPORTED, "head_dim %d: only 64 and 128 are built", c->head_dim);
  if (c->chunk_size != hils::kChunk)
    return fail(HILS_ERR_UNSUPPORTED, "chunk_size %d: only 64 is built", c->chunk_size);
  if (c->top_k < 1 || c->top_k > hils::kMaxTopK)
    return fail(HILS_ERR_INVALID_ARG, "top_k %d outside 1..%d", c->top_k, hils::kMaxTopK);
  if (c->calib_rank < 0 || c->calib_rank > hils::kMaxRank)
    return fail(HILS_ERR_INVALID_ARG, "calib_rank %d outside 0..%d", c->calib_rank, hils::kMaxRank);
  if (c->dtype != HILS_F32 && c->dtype != HILS_BF16)
    return fail(HILS_ERR_INVALID_ARG, "dtype %d is neither HILS_F32 nor HILS_BF16", c->dtype);
  hils::Params p{};
  p.B = c->batch;
  p.Hq = c->n_q_heads;
  p.Hkv = c->n_kv_heads;
  p.d = c->head_dim;
  p.k = c->top_k;
  p.r = c->calib_rank;
  p.dtype = c->dtype;
  p.group = c->n_q_heads / c->n_kv_heads;
  p.inv_sqrt_d = (float)(1.0 / std::sqrt((double)c->head_dim));
  *P = p;
  return HILS_OK;
}

int check_calib(const hils_config* c, const float* A, const float* B, hils::Params* P) {
  if (c->calib_rank > 0 && (!A || !B))
    return fail(HILS_ERR_INVALID_ARG, "calib_rank %d needs A and B", c->calib_rank);
  if (c->calib_rank > 0 && (!aligned16(A) || !aligned16(B)))
    return fail(HILS_ERR_INVALID_ARG, "A and B must be 16-byte aligned");
  P->A = A;
  P->Bm = B;
  return HILS_OK;
}

int check_landmarks(const hils_kv_cache* kc, hils::Params* P) {
  if (!kc) return fail(HILS_ERR_INVALID_ARG, "cache is NULL");
  if (!kc->landmarks) return fail(HILS_ERR_INVALID_ARG, "cache->landmarks is NULL");
  if (!aligned16(kc->landmarks)) return fail(HILS_ERR_INVALID_ARG, "landmarks not 16-byte aligned");
  if (kc->max_chunks <= 0) return fail(HILS_ERR_INVALID_ARG, "max_chunks must be positive");
  P->landmarks = kc->landmarks;
  P->max_chunks = kc->max_chunks;
  return HILS_OK;
}

int check_pages(const hils_kv_cache* kc, hils::Params* P) {
  int st = check_landmarks(kc, P);
  if (st) return st;
  if (!kc->pages || !kc->block_table)
    return fail(HILS_ERR_INVALID_ARG, "cache->pages and cache->block_table are required");
  if (!aligned16(kc->pages)) return fail(HILS_ERR_INVALID_ARG, "pages not 16-byte aligned");
  if (kc->num_pages <= 0) return fail(HILS_ERR_INVALID_ARG, "num_pages must be positive");
  P->pages = kc->pages;
  P->num_pages = kc->num_pages;
  P->block_table = kc->block_table;
  P->seq_lens = kc->seq_lens;
  return HILS_OK;
}

int check_queries(const void* q, int64_t q_len, int64_t q_pos0, const hils::Params& P,
                  int32_t n_chunks_limit) {
  if (!q) return fail(HILS_ERR_INVALID_ARG, "q is NULL");
  if (!aligned16(q)) return fail(HILS_ERR_INVALID_ARG, "q not 16-byte aligned");
  if (q_len < 0 || q_pos0 < 0) return fail(HILS_ERR_INVALID_ARG, "q_len and q_pos0 must be >= 0");
  if (q_len > 0 && (q_pos0 + q_len - 1) / hils::kChunk >= n_chunks_limit)
    return fail(HILS_ERR_INVALID_ARG,
                "last query position %lld lies in chunk %lld, beyond the %d chunks available",
                (long long)(q_pos0 + q_len - 1), (long long)((q_pos0 + q_len - 1) / hils::kChunk),
                n_chunks_limit);
  const int64_t pairs = (int64_t)P.B * q_len * P.Hq * P.k;
  if (pairs >= ((int64_t)1 << 31))
    return fail(HILS_ERR_UNSUPPORTED, "B*q_len*Hq*top_k = %lld exceeds 2^31-1", (long long)pairs);
  return HILS_OK;
}

}  // namespace

extern "C" {

size_t hils_workspace_size(const hils_config* cfg, int op, int64_t q_len, int32_t max_chunks) {
  hils::Params P{};
  if (check_config(cfg, &P) != HILS_OK) return 0;
  if (q_len < 0 || max_chunks <= 0) {
    fail(HILS_ERR_INVALID_ARG, "q_len must be >= 0 and max_chunks positive");
    return 0;
  }
  P.L = q_len;
  P.max_chunks = max_chunks;
  switch (op) {
    case HILS_OP_SCORE:
    case HILS_OP_TOPK:
      return 0;
    case HILS_OP_PREFILL:
      return hils::prefill_ws_bytes(P, nullptr, nullptr);
    case HILS_OP_DECODE:
      return hils::decode_ws_bytes(P, nullptr, nullptr);
    case HILS_OP_PREFILL_BACKWARD:
      return hils::backward_ws_bytes(P, nullptr, nullptr);
    default:
      fail(HILS_ERR_INVALID_ARG, "unknown op %d", op);
      return 0;
  }
}

int hils_score(const hils_config* cfg, const void* q, int64_t q_len, int64_t q_pos0,
               const float* A, const float* B, const hils_kv_cache* cache, float* scores,
               int32_t n_cols, void* stream) {
  hils::Params P{};
  int st;
  if ((st = check_config(cfg, &P)) || (st = check_calib(cfg, A, B, &P)) ||
      (st = check_landmarks(cache, &P)))
    return st;
  if (!scores) return fail(HILS_ERR_INVALID_ARG, "scores is NULL");
  if (n_cols <= 0 || n_cols > cache->max_chunks)
    return fail(HILS_ERR_INVALID_ARG, "n_cols %d outside 1..max_chunks", n_cols);
  if ((st = check_queries(q, q_len, q_pos0, P, n_cols))) return st;
  P.q = q;
  P.L = q_len;
  P.pos0 = q_pos0;
  cudaError_t e = hils::launch_score(P, scores, n_cols, (cudaStream_t)stream);
  return e == cudaSuccess ? HILS_OK : cuda_fail(e, "hils_score");
}

int hils_topk(const hils_config* cfg, const float* scores, int64_t q_len, int64_t q_pos0,
              int32_t n_cols, int32_t* idx, float* w, void* stream) {
  hils::Params P{};
  int st;
  if ((st = check_config(cfg, &P))) return st;
  if (!scores || !idx || !w) return fail(HILS_ERR_INVALID_ARG, "scores, idx and w are required");
  if (n_cols <= 0) return fail(HILS_ERR_INVALID_ARG, "n_cols must be positive");
  if (q_len < 0 || q_pos0 < 0) return fail(HILS_ERR_INVALID_ARG, "q_len and q_pos0 must be >= 0");
  if (q_len > 0 && (q_pos0 + q_len - 1) / hils::kChunk >= n_cols)
    return fail(HILS_ERR_INVALID_ARG, "own chunk of the last query is beyond n_cols");
  P.L = q_len;
  P.pos0 = q_pos0;
  cudaError_t e = hils::launch_topk(P, scores, n_cols, idx, w, (cudaStream_t)stream);
  return e == cudaSuccess ? HILS_OK : cuda_fail(e, "hils_topk");
}

int hils_prefill(const hils_config* cfg, const void* q, int64_t q_len, int64_t q_pos0,
                 const float* A, const float* B, const hils_kv_cache* cache, void* out,
                 int32_t* idx_out, float* w_out, void* ws, size_t ws_bytes, void* stream) {
  hils::Params P{};
  int st;
  if ((st = check_config(cfg, &P)) || (st = check_calib(cfg, A, B, &P)) ||
      (st = check_pages(cache, &P)))
    return st;
  if ((st = check_queries(q, q_len, q_pos0, P, cache->max_chunks))) return st;
  if (!out || !aligned16(out)) return fail(HILS_ERR_INVALID_ARG, "out is NULL or misaligned");
  P.q = q;
  P.L = q_len;
  P.pos0 = q_pos0;
  hils::PrefillWs w{};
  const size_t need = hils::prefill_ws_bytes(P, &w, nullptr);
  if (!ws || ws_bytes < need)
    return fail(HILS_ERR_WORKSPACE, "prefill needs %zu workspace bytes, got %zu", need, ws_bytes);
  if (((uintptr_t)ws & 255u) != 0) return fail(HILS_ERR_INVALID_ARG, "workspace not 256-byte aligned");
  hils::prefill_ws_bytes(P, &w, (char*)ws);
  cudaError_t e = hils::launch_prefill(P, out, idx_out, w_out, w, (cudaStream_t)stream);
  return e == cudaSuccess ? HILS_OK : cuda_fail(e, "hils_prefill");
}

int hils_prefill_backward(const hils_config* cfg, const void* q, int64_t q_len, int64_t q_pos0,
                          const float* A, const float* B, const hils_kv_cache* cache,
                          const int32_t* idx, const float* w, const void* out,
                          const void* dout, float* dq, float* dpages, float* dlandmarks,
                          float* dA, float* dB, void* ws, size_t ws_bytes, void* stream) {
  hils::Params P{};
  int st;
  if ((st = check_config(cfg, &P)) || (st = check_calib(cfg, A, B, &P)) ||
      (st = check_pages(cache, &P)))
    return st;
  if ((st = check_queries(q, q_len, q_pos0, P, cache->max_chunks))) return st;
  if (!idx || !w) return fail(HILS_ERR_INVALID_ARG, "idx and w (the forward's selection) are required");
  if (!dout || !aligned16(dout)) return fail(HILS_ERR_INVALID_ARG, "dout is NULL or misaligned");
  if (!out || !aligned16(out)) return fail(HILS_ERR_INVALID_ARG, "out is NULL or misaligned");
  if (!dq || !dpages || !dlandmarks)
    return fail(HILS_ERR_INVALID_ARG, "dq, dpages and dlandmarks are required");
  if (!aligned16(dq)) return fail(HILS_ERR_INVALID_ARG, "dq not 16-byte aligned");
  if (P.r > 0 && (!dA || !dB)) return fail(HILS_ERR_INVALID_ARG, "dA and dB are required when calib_rank > 0");
  P.q = q;
  P.L = q_len;
  P.pos0 = q_pos0;
  hils::BackwardWs w_ws{};
  const size_t need = hils::backward_ws_bytes(P, &w_ws, nullptr);
  if (!ws || ws_bytes < need)
    return fail(HILS_ERR_WORKSPACE, "prefill backward needs %zu workspace bytes, got %zu", need,
                ws_bytes);
  if (((uintptr_t)ws & 255u) != 0) return fail(HILS_ERR_INVALID_ARG, "workspace not 256-byte aligned");
  hils::backward_ws_bytes(P, &w_ws, (char*)ws);
  cudaError_t e = hils::launch_backward(P, idx, w, out, dout, dq, dpages, dlandmarks, dA, dB,
                                        w_ws, (cudaStream_t)stream);
  return e == cudaSuccess ? HILS_OK : cuda_fail(e, "hils_prefill_backward");
}

int hils_decode(const hils_config* cfg, const void* q, const void* k_new, const void* v_new,
                const float* A, const float* B, hils_kv_cache* cache, void* out, int32_t* idx_out,
                float* w_out, void* ws, size_t ws_bytes, void* stream) {
  return hils::decode_call(cfg, q, k_new, v_new, A, B, cache, out, idx_out, w_out, ws, ws_bytes,
                           false, stream);
}

namespace {
// Lays the decode scratch out at `ws` after checking that the configuration
// fits the kernels and that the buffer is large enough and 256-byte aligned.
int decode_layout(const hils::Params& P, void* ws, size_t ws_bytes, hils::DecodeWs* w) {
  if (P.Hq > 64) return fail(HILS_ERR_UNSUPPORTED, "decode supports up to 64 query heads");
  const size_t need = hils::decode_ws_bytes(P, w, nullptr);
  if (w->n_split > hils::kMaxSplitLists)
    return fail(HILS_ERR_UNSUPPORTED, "decode supports up to %d chunk ranges (max_chunks %d needs %d)",
                hils::kMaxSplitLists, P.max_chunks, w->n_split);
  if (hils::decode_smem_bytes(P, *w) > 227 * 1024)
    return fail(HILS_ERR_UNSUPPORTED,
                "decode of %d query heads per KV head over %d chunk ranges needs more shared "
                "memory than a CTA has", P.group, w->n_split);
  if (!ws || ws_bytes < need)
    return fail(HILS_ERR_WORKSPACE, "decode needs %zu workspace bytes, got %zu", need, ws_bytes);
  if (((uintptr_t)ws & 255u) != 0) return fail(HILS_ERR_INVALID_ARG, "workspace not 256-byte aligned");
  hils::decode_ws_bytes(P, w, (char*)ws);
  return HILS_OK;
}
}  // namespace

// ---- context-parallel decode ----
namespace {
int cp_common(const hils_config* cfg, const void* q, const void* k_new, const void* v_new,
              hils::Params* P) {
  if (!q || !aligned16(q)) return fail(HILS_ERR_INVALID_ARG, "q is NULL or misaligned");
  if ((k_new == nullptr) != (v_new == nullptr))
    return fail(HILS_ERR_INVALID_ARG, "k_new and v_new must both be given or both be NULL");
  if (k_new && (!aligned16(k_new) || !aligned16(v_new)))
    return fail(HILS_ERR_INVALID_ARG, "k_new and v_new must be 16-byte aligned");
  P->q = q;
  P->L = 1;
  return HILS_OK;
}
}  // namespace

int hils_decode_cp_candidates(const hils_config* cfg, const void* q, const void* k_new,
                              const void* v_new, const float* A, const float* B,
                              hils_kv_cache* shard, int64_t chunk_base, uint64_t* keys,
                              float* own_score, void* ws, size_t ws_bytes, void* stream) {
  hils::Params P{};
  int st;
  if ((st = check_config(cfg, &P)) || (st = check_calib(cfg, A, B, &P)) ||
      (st = check_pages(shard, &P)) || (st = cp_common(cfg, q, k_new, v_new, &P)))
    return st;
  if (!shard->seq_lens) return fail(HILS_ERR_INVALID_ARG, "shard->seq_lens is required");
  if (chunk_base < 0) return fail(HILS_ERR_INVALID_ARG, "chunk_base must be >= 0");
  if ((cfg->top_k > 1 && !keys) || !own_score)
    return fail(HILS_ERR_INVALID_ARG, "keys and own_score are required");
  hils::DecodeWs w{};
  if ((st = decode_layout(P, ws, ws_bytes, &w))) return st;
  w.chunk_base = chunk_base;
  w.cp_keys = keys;
  w.cp_own = own_score;
  if (P.B == 0) return HILS_OK;
  cudaError_t e = hils::launch_cp_candidates(P, k_new, v_new, w, (cudaStream_t)stream);
  return e == cudaSuccess ? HILS_OK : cuda_fail(e, "hils_decode_cp_candidates");
}

int hils_decode_cp_select(const hils_config* cfg, int32_t world, const uint64_t* keys,
                          const float* own_scores, const int32_t* seq_lens, int32_t append,
                          int32_t* idx, float* w, void* stream) {
  hils::Params P{};
  int st;
  if ((st = check_config(cfg, &P))) return st;
  if (world < 1) return fail(HILS_ERR_INVALID_ARG, "world must be positive");
  if ((cfg->top_k > 1 && !keys) || !own_scores || !seq_lens || !idx || !w)
    return fail(HILS_ERR_INVALID_ARG, "keys, own_scores, seq_lens, idx and w are required");
  P.seq_lens = const_cast<int32_t*>(seq_lens);
  if (P.B == 0) return HILS_OK;
  cudaError_t e = hils::launch_cp_select(P, world, keys, own_scores, append != 0, idx, w,
                                         (cudaStream_t)stream);
  return e == cudaSuccess ? HILS_OK : cuda_fail(e, "hils_decode_cp_select");
}

int hils_decode_cp_attend(const hils_config* cfg, const void* q, const void* k_new,
                          const void* v_new, const hils_kv_cache* shard, int64_t chunk_base,
                          const int32_t* idx, const float* w, float* partial, void* stream) {
  hils::Params P{};
  int st;
  if ((st = check_config(cfg, &P)) || (st = check_pages(shard, &P)) ||
      (st = cp_common(cfg, q, k_new, v_new, &P)))
    return st;
  if (!shard->seq_lens) return fail(HILS_ERR_INVALID_ARG, "shard->seq_lens is required");
  if (chunk_base < 0) return fail(HILS_ERR_INVALID_ARG, "chunk_base must be >= 0");
  if (!idx || !w || !partial) return fail(HILS_ERR_INVALID_ARG, "idx, w and partial are required");
  if (P.B == 0) return HILS_OK;
  cudaError_t e = hils::launch_cp_attend(P, chunk_base, k_new, v_new, idx, w, partial,
                                         (cudaStream_t)stream);
  return e == cudaSuccess ? HILS_OK : cuda_fail(e, "hils_decode_cp_attend");
}

int hils_decode_cp_finish(const hils_config* cfg, const float* sum, void* out, int32_t* seq_lens,
                          int32_t append, void* stream) {
  hils::Params P{};
  int st;
  if ((st = check_config(cfg, &P))) return st;
  if (!sum || !out) return fail(HILS_ERR_INVALID_ARG, "sum and out are required");
  if (append && !seq_lens) return fail(HILS_ERR_INVALID_ARG, "seq_lens is required to append");
  P.seq_lens = seq_lens;
  if (P.B == 0) return HILS_OK;
  cudaError_t e = hils::launch_cp_finish(P, sum, out, append != 0, (cudaStream_t)stream);
  return e == cudaSuccess ? HILS_OK : cuda_fail(e, "hils_decode_cp_finish");
}

int hils_device_status(void* stream) {
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "hils_device_status: stream synchronize");
  int word = 0;
  e = cudaMemcpyFromSymbol(&word, hils::g_device_error, sizeof word);
  if (e != cudaSuccess) return cuda_fail(e, "hils_device_status: read");
  if (word == 0) return HILS_OK;
  const int zero = 0;
  e = cudaMemcpyToSymbol(hils::g_device_error, &zero, sizeof zero);
  if (e != cudaSuccess) return cuda_fail(e, "hils_device_status: clear");
  return fail((word & hils::kErrTimeout) ? HILS_ERR_TIMEOUT : HILS_ERR_DEVICE_CHECK,
              "device check fired (bits 0x%x: %s%s%s)", word,
              (word & hils::kErrPage) ? "page " : "", (word & hils::kErrChunk) ? "chunk " : "",
              (word & hils::kErrTimeout) ? "a bounded wait ran out" : "");
}

int hils_set_wait_limit_ns(uint64_t ns) {
  const uint64_t v = ns == 0 ? hils::kDrainLimitNs : ns;
  cudaError_t e = cudaMemcpyToSymbol(hils::g_wait_limit_ns, &v, sizeof v);
  return e == cudaSuccess ? HILS_OK : cuda_fail(e, "hils_set_wait_limit_ns");
}

const char* hils_last_error(void) { return g_last_error.c_str(); }

const char* hils_version(void) { return "hils-b200 0.1.0 sm_100a"; }

}  // extern "C"

namespace hils {
// Lets other translation units of the library report through hils_last_error().
void record_error(const char* msg) { g_last_error = msg; }

cudaError_t set_smem_impl(const void* func, size_t bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, size_t> done;
  std::lock_guard<std::mutex> lock(mu);
  size_t& have = done[{func, dev}];
  if (have >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess) have = bytes;
  return e;
}
}  // namespace hils

namespace hils {
int decode_call(const hils_config* cfg, const void* q, const void* k_new, const void* v_new,
                const float* A, const float* B, hils_kv_cache* cache, void* out, int32_t* idx_out,
                float* w_out, void* ws, size_t ws_bytes, bool clear_counters, void* stream) {
  Params P{};
  int st;
  if ((st = check_config(cfg, &P)) || (st = check_calib(cfg, A, B, &P)) ||
      (st = check_pages(cache, &P)))
    return st;
  if (!q || !aligned16(q)) return fail(HILS_ERR_INVALID_ARG, "q is NULL or misaligned");
  if (!out) return fail(HILS_ERR_INVALID_ARG, "out is NULL");
  if ((k_new == nullptr) != (v_new == nullptr))
    return fail(HILS_ERR_INVALID_ARG, "k_new and v_new must both be given or both be NULL");
  if (k_new && (!aligned16(k_new) || !aligned16(v_new)))
    return fail(HILS_ERR_INVALID_ARG, "k_new and v_new must be 16-byte aligned");
  if (!cache->seq_lens) return fail(HILS_ERR_INVALID_ARG, "cache->seq_lens is required for decode");
  P.q = q;
  P.L = 1;
  P.pos0 = 0;
  DecodeWs w{};
  if ((st = decode_layout(P, ws, ws_bytes, &w))) return st;
  if (P.B == 0) return HILS_OK;
  cudaError_t e;
  if (clear_counters &&
      (e = cudaMemsetAsync(w.tickets, 0, w.ticket_bytes, (cudaStream_t)stream)) != cudaSuccess)
    return cuda_fail(e, "clearing the completion counters");
  e = launch_decode(P, k_new, v_new, out, idx_out, w_out, w, (cudaStream_t)stream);
  return e == cudaSuccess ? HILS_OK : cuda_fail(e, "hils_decode");
}
}  // namespace hils
