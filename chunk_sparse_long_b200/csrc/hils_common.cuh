// Internal declarations shared by the HiLS CUDA kernels and the C-ABI layer.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/hils.h"

namespace hils {

constexpr int kChunk = 64;       // chunk_size the kernels are written for
constexpr int kItemPairs = 512;  // pairs per tensor-core attention work item (4 tiles of 128)
constexpr int kMaxTopK = 32;
constexpr int kMaxRank = 64;
constexpr int kMaxSplitLists = 512;  // decode: chunk ranges per (sequence, KV head), at most
constexpr int kScoreTileRows = 128;  // query rows per landmark-scoring tile
constexpr int kScoreBlock = 128;     // landmark chunks per scoring block

// Tile t of 128 query rows sees score_tile_blocks(t) blocks of 128 landmark
// chunks (enough for the last causally visible chunk of its last row).
__host__ __device__ inline int64_t score_tile_blocks(int64_t L, int64_t pos0, int64_t t) {
  const int64_t last = (t + 1) * kScoreTileRows < L ? (t + 1) * kScoreTileRows - 1 : L - 1;
  return (pos0 + last) / ((int64_t)kChunk * kScoreBlock) + 1;
}

// Device error word: kernels OR bits into it when a bounds check fires.
enum DeviceError : int {
  kErrPage = 1,      // block_table entry outside [0, num_pages)
  kErrChunk = 2,     // selected chunk index outside [0, max_chunks)
  kErrTimeout = 4,   // a bounded wait ran out
};
extern __device__ int g_device_error;

__device__ __forceinline__ void set_device_error(int bit) { atomicOr(&g_device_error, bit); }

// How long a kernel's waits on its pipeline (one stage waiting for another)
// last before the kernel gives up and reports a timeout: 2 s unless a test
// lowers it (hils_set_wait_limit_ns).  The waits that let a kernel's own
// asynchronous copies and products finish before it exits always use
// kDrainLimitNs, so that a kernel that gives up never leaves work in flight.
extern __constant__ uint64_t g_wait_limit_ns;
constexpr uint64_t kDrainLimitNs = 2000000000ull;
__device__ __forceinline__ uint64_t wait_limit() { return g_wait_limit_ns; }

// Plain parameters of one call, passed by value to every kernel.
struct Params {
  int B, Hq, Hkv, d, k, r, dtype;
  int group;              // Hq / Hkv
  float inv_sqrt_d;
  const void* q;          // prefill [B][L][Hq][d]; decode [B][Hq][d]
  int64_t L, pos0;
  const float* A;         // [d][r]
  const float* Bm;        // [r][d]
  const void* pages;
  int64_t num_pages;
  const int32_t* block_table;
  int max_chunks;
  const void* landmarks;
  int32_t* seq_lens;
};

// ---- storage loads ------------------------------------------------------
__device__ __forceinline__ float bf16_to_f32(uint16_t b) {
  return __uint_as_float(((uint32_t)b) << 16);
}

__device__ __forceinline__ float load_elem(const void* p, int dtype, int64_t i) {
  if (dtype == HILS_F32) return ((const float*)p)[i];
  return bf16_to_f32(((const uint16_t*)p)[i]);
}

// Eight consecutive elements starting at element i (i a multiple of 8, 16-byte aligned).
__device__ __forceinline__ void load8(const void* p, int dtype, int64_t i, float* v) {
  if (dtype == HILS_F32) {
    const float4* f = reinterpret_cast<const float4*>((const float*)p + i);
    float4 a = f[0], b = f[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  } else {
    uint4 u = *reinterpret_cast<const uint4*>((const uint16_t*)p + i);
    uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      v[2 * a] = __uint_as_float(w[a] << 16);
      v[2 * a + 1] = __uint_as_float(w[a] & 0xFFFF0000u);
    }
  }
}

__device__ __forceinline__ void store_elem(void* p, int dtype, int64_t i, float v) {
  if (dtype == HILS_F32)
    ((float*)p)[i] = v;
  else
    ((__nv_bfloat16*)p)[i] = __float2bfloat16_rn(v);
}

// Element offset of (page, kind, kv head g, slot s, element 0) in the page pool.
__device__ __forceinline__ int64_t page_offset(const Params& P, int64_t page, int kind, int g,
                                               int s) {
  return (((page * 2 + kind) * P.Hkv + g) * (int64_t)kChunk + s) * P.d;
}

// Physical page of logical chunk j of sequence b, or -1 (and the error bit) if
// the block table points outside the pool.
__device__ __forceinline__ int64_t page_of(const Params& P, int b, int64_t j) {
  if (j < 0 || j >= P.max_chunks) {
    set_device_error(kErrChunk);
    return -1;
  }
  int64_t page = P.block_table[(int64_t)b * P.max_chunks + j];
  if (page < 0 || page >= P.num_pages) {
    set_device_error(kErrPage);
    return -1;
  }
  return page;
}

// RAII bracket of one kernel launch for the optional event profiler
// (hils_profile_enable); a no-op unless profiling is on.
class ProfileScope {
 public:
  ProfileScope(const char* phase, cudaStream_t s);
  ~ProfileScope();

 private:
  const char* phase_;
  cudaStream_t stream_;
  void* start_ = nullptr;
};
#define HILS_PROFILE(name, stream) ::hils::ProfileScope _hils_prof_scope_(name, stream)

// Sets the message hils_last_error() returns on this thread.
void record_error(const char* msg);

// Raises a kernel's dynamic shared-memory limit to `bytes` on the current
// device, calling the runtime only the first time a larger value is needed.
cudaError_t set_smem_impl(const void* func, size_t bytes);
template <typename F>
cudaError_t set_smem(F* func, size_t bytes) {
  return set_smem_impl(reinterpret_cast<const void*>(func), bytes);
}

// Tensor map of a bf16 tensor with `rank` (2..5) dimensions, innermost first:
// dims[x] elements along dimension x, strides[x] bytes from one index of
// dimension x + 1 to the next (rank - 1 of them), box[x] elements per copy;
// 128-byte swizzle, elements outside the tensor read as zeros.
cudaError_t encode_tmap_bf16(CUtensorMap* tm, int rank, const void* base, const uint64_t* dims,
                             const uint64_t* strides, const uint32_t* box);
// The same for a tensor of `dtype` (HILS_BF16 or HILS_F32).
cudaError_t encode_tmap(CUtensorMap* tm, int dtype, int rank, const void* base,
                        const uint64_t* dims, const uint64_t* strides, const uint32_t* box);

// ---- launchers (each returns cudaError_t of its launches) -----------------
cudaError_t launch_score(const Params& P, float* scores, int n_cols, cudaStream_t s);
cudaError_t launch_topk(const Params& P, const float* scores, int n_cols, int32_t* idx, float* w,
                        cudaStream_t s);

struct PrefillWs {
  int32_t* idx;      // [rows][k]
  float* w;          // [rows][k]
  int32_t* counts;   // [n_keys]; key = ((b * Hkv + g) * n_win + window) * max_chunks + chunk
  int32_t* offsets;  // [n_keys + 1] pair offsets
  int32_t* tile_off; // [n_keys + 1] tile offsets
  int32_t* cursor;   // [n_keys]
  int32_t* pairs;    // float32 path: [rows * k] pair ids (row * k + slot) in bucket order
  int2* pinfo;       // bf16 path: [rows * k] (query row, fusion weight bits with the visible
                     // keys - 1 in the 6 lowest) in bucket order
  float* acc;        // [rows][d] float32 accumulator (CUDA-core attention)
  void* qimg;        // bf16: per 128-row tile the three q~ term tiles (shared-memory images)
  int4* items;       // [max_tiles] (key, first pair, end pair, 0) of every work item
  int2* scan_totals; // [ceil(n_keys / 1024)] (pairs, items) of each block of keys
  int n_keys;
  int n_win;         // query windows per sequence
  int64_t win_rows;  // query positions per window
  int64_t max_tiles;
};
size_t prefill_ws_bytes(const Params& P, PrefillWs* ws, char* base);
// Key-major bucketing of the (row, slot) pairs of idx [B][L][Hq][k] by
// (sequence, KV head, query window, chunk) into ws: counts, offsets, the work
// items (up to tile_pairs pairs of one key each) and, per pair in bucket
// order, either its id row * k + slot (ws.pairs) or, with records, its
// tensor-core record (ws.pinfo).
cudaError_t launch_bucketing(const Params& P, const int32_t* idx, const float* w,
                             const PrefillWs& ws, bool records, int tile_pairs, const char* label,
                             cudaStream_t s);

// Prefill backward with the selection fixed (hils_prefill_backward).
constexpr int kBackwardTilePairs = 128;
constexpr int kBackwardMaxCtas = 160;   // per-CTA partial sums of the tensor-core path
// True where the attention part runs on the tensor cores (bf16, head_dim 128).
inline bool backward_on_tc(const Params& P) { return P.dtype == HILS_BF16 && P.d == 128; }
struct BackwardWs {
  PrefillWs bk;     // bucketing: pair ids in key order, items of kBackwardTilePairs pairs
  float* dw;        // CUDA-core path: [rows * k] dout . O_j per pair
  float* delta;     // tensor-core path: [rows] dout . out per row
  float* lmc;       // tensor-core path: [B][max_chunks][Hkv][d] lm + (lm B^T) A^T
  float* vchunk;    // tensor-core path: [B][max_chunks][Hkv][d] sum over chunk j's pairs of ds q
  float* mpart;     // tensor-core path: [kBackwardMaxCtas + 1][d][d] per-CTA sums of v lm^T
};
// Workspace carve-up; with base == nullptr only the size is computed.
size_t backward_ws_bytes(const Params& P, BackwardWs* ws, char* base);
cudaError_t launch_backward(const Params& P, const int32_t* idx, const float* w, const void* out,
                            const void* dout, float* dq, float* dpages, float* dlm, float* dA,
                            float* dB, const BackwardWs& ws, cudaStream_t s);
// The tensor-core path after the bucketing: everything but the bucketing.
cudaError_t launch_backward_tc(const Params& P, const int32_t* idx, const float* w,
                               const void* out, const void* dout, float* dq, float* dpages,
                               float* dlm, float* dA, float* dB, const BackwardWs& ws,
                               cudaStream_t s);
cudaError_t launch_prefill(const Params& P, void* out, int32_t* idx_out, float* w_out,
                           const PrefillWs& ws, cudaStream_t s);
cudaError_t launch_select_tc(const Params& P, const PrefillWs& ws, int32_t* idx, float* w,
                             cudaStream_t s);
cudaError_t launch_attn_tc(const Params& P, void* out, const PrefillWs& ws, cudaStream_t s);

struct DecodeWs {
  uint64_t* cand;      // [B][Hq][n_split][k-1] each range's best candidates as selection keys,
                       // best first
  int32_t* idx;        // [B][Hq][k] selected chunks (slot 0 = own)
  float* w;            // [B][Hq][k] fusion weights
  int32_t* page;       // [B][Hq][k] their pages (-1: none)
  int32_t* tickets;    // [B][Hkv] scan tickets, then [B] heads done; all return to zero
                       // at the end of every step
  size_t ticket_bytes;
  int n_split, chunks_per_split;
  int append;          // k_new / v_new given
  // context-parallel mode (cp_keys or cp_partial set): the cache holds the
  // chunks chunk_base .. chunk_base + max_chunks - 1 of every sequence and
  // seq_lens the global positions.  The scan then leaves the merged keys
  // [B][Hq][k-1] and the own chunk's score [B][Hq] (-inf where not held)
  // instead of the weights; the attention reads idx and w (global chunks),
  // looks the pages up itself and writes float32 weighted sums to cp_partial
  // without advancing seq_lens.
  int64_t chunk_base;
  uint64_t* cp_keys;
  float* cp_own;
  float* cp_partial;
};
size_t decode_ws_bytes(const Params& P, DecodeWs* ws, char* base);
// Dynamic shared memory of the decode kernel for this configuration.
size_t decode_smem_bytes(const Params& P, const DecodeWs& ws);
// hils_decode with its scratch at `ws`: validates every argument, lays the
// workspace out, then (clear_counters) zeroes its completion counters on the
// stream and launches the step.  Nothing is queued when a check fails.
int decode_call(const hils_config* cfg, const void* q, const void* k_new, const void* v_new,
                const float* A, const float* B, hils_kv_cache* cache, void* out, int32_t* idx_out,
                float* w_out, void* ws, size_t ws_bytes, bool clear_counters, void* stream);
cudaError_t launch_decode(const Params& P, const void* k_new, const void* v_new, void* out,
                          int32_t* idx_out, float* w_out, const DecodeWs& ws, cudaStream_t s);

// Context-parallel decode (this GPU holds chunks chunk_base .. chunk_base +
// P.max_chunks - 1 of every sequence); see hils_decode_cp_* in hils.h.
// The scan over this GPU's chunks; ws laid out by decode_ws_bytes for the
// shard, with chunk_base, cp_keys and cp_own set.
cudaError_t launch_cp_candidates(const Params& P, const void* k_new, const void* v_new,
                                 const DecodeWs& ws, cudaStream_t s);
cudaError_t launch_cp_select(const Params& P, int world, const uint64_t* keys,
                             const float* own_scores, bool append, int32_t* idx, float* w,
                             cudaStream_t s);
cudaError_t launch_cp_attend(const Params& P, int64_t chunk_base, const void* k_new,
                             const void* v_new, const int32_t* idx, const float* w, float* partial,
                             cudaStream_t s);
cudaError_t launch_cp_finish(const Params& P, const float* sum, void* out, bool append,
                             cudaStream_t s);

}  // namespace hils
