// Prefill per-chunk attention (a5) and fused merge (a6) on the 5th-generation
// tensor cores (tcgen05, TMEM accumulators), bf16 inputs.
//
// Work is key-major: the (row, slot) pairs are bucketed by (sequence, KV head,
// chunk) and a work item is up to kItemPairs pairs of one bucket, so the
// chunk's 64 x d K and V tiles are staged in shared memory once per item and
// shared by up to four 128-row tiles.  Per 128-row tile:
//
//   gather   every thread copies its pair's query row (cp.async, 16 B) into a
//            128-byte-swizzled K-major tile; the next tile's rows are
//            prefetched into the other buffer while this one is computed
//   S = Q K^T   tcgen05.mma, M=128 N=64, f32 in TMEM
//   softmax  thread t reads TMEM lane t (its pair's 64 logits), masks keys
//            after the query in the own chunk, writes P (bf16) over the
//            consumed Q tile
//   O = P V  tcgen05.mma, M=128 N=d, V read MN-major from the same tile
//   epilogue O * (w / l) -> bf16 partial, staged in shared memory and written
//            row-contiguously to partial[pair] (one 2d-byte row per pair)
//
// merge_kernel then sums each query row's k partials in float32 (slot order,
// deterministic) and writes the output row.  Partials are rounded to bf16 once
// each, relative to their own (small) magnitude.
#include <cfloat>

#include "hils_common.cuh"
#include "tc_common.cuh"

namespace hils {
namespace {

constexpr int kRows = 128;          // pairs per MMA tile (M)
constexpr int kThreads = 128;       // one thread per tile row / TMEM lane
constexpr uint32_t kTmemCols = 256; // S (64 cols) + O (d cols)

template <int D>
struct AttnLayout {
  static constexpr uint32_t kQBytes = kRows * D * 2;   // one query tile
  static constexpr uint32_t kKVBytes = kChunk * D * 2; // one K (or V) tile
  static constexpr uint32_t kQ0 = 0;
  static constexpr uint32_t kQ1 = kQBytes;
  static constexpr uint32_t kK = 2 * kQBytes;
  static constexpr uint32_t kV = kK + kKVBytes;
  static constexpr uint32_t kEnd = kV + kKVBytes;
  // + slack for 1024-byte alignment; at least the d=128 footprint so that no more
  // than two CTAs share an SM (two CTAs x 256 TMEM columns = the SM's 512)
  static constexpr uint32_t kSmem = (kEnd + 1024 > 99328u) ? kEnd + 1024 : 99328u;
};

__device__ __forceinline__ int find_key(const int32_t* tile_off, int n_keys, int item) {
  int lo = 0, hi = n_keys - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (tile_off[mid] <= item) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Copy one query row (pair id pid, or zeros when pid < 0) into tile buffer q_smem.
template <int D>
__device__ __forceinline__ void gather_q_row(const Params& P, uint32_t q_smem, int row, int32_t pid) {
  const int64_t r = pid >= 0 ? pid / P.k : 0;
  const uint16_t* src = reinterpret_cast<const uint16_t*>(P.q) + r * D;
  const uint32_t bytes = pid >= 0 ? 16u : 0u;
#pragma unroll
  for (int c = 0; c < D / 8; ++c) {
    const uint32_t dst = q_smem + (uint32_t)(c >> 3) * (kRows * 128) + tc::swz(row, c & 7);
    tc::cp_async16(dst, src + c * 8, bytes);
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 2) attn_tc_kernel(Params P, PrefillWs ws) {
  using Lay = AttnLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bar_s, bar_o;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int item_sh;
  __shared__ int abort_sh;
  __shared__ int32_t pid_sh[kRows];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~(uintptr_t)1023);
  const uint32_t sbase = tc::smem_u32(smem);
  const int tid = threadIdx.x, warp = tid >> 5;

  if (tid == 0) {
    tc::mbar_init(&bar_s, 1);
    tc::mbar_init(&bar_o, 1);
    tc::fence_mbar_init();
    abort_sh = 0;
  }
  if (warp == 0) {
    tc::tmem_alloc(&tmem_base_sh, kTmemCols);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  const uint32_t tmem_s = tmem;          // columns [0, 64)
  const uint32_t tmem_o = tmem + 64;     // columns [64, 64 + D)
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
  constexpr uint32_t kIdS = tc::idesc_bf16(kRows, kChunk, 0);
  constexpr uint32_t kIdO = tc::idesc_bf16(kRows, D, 1);
  const float scale_log2 = P.inv_sqrt_d * 1.4426950408889634f;

  uint32_t phase_s = 0, phase_o = 0;
  const int n_items = ws.tile_off[ws.n_keys];
  int prev_key = -1;

  for (;;) {
    if (tid == 0) item_sh = atomicAdd(ws.queue, 1);
    __syncthreads();
    const int item = item_sh;
    if (item >= n_items || abort_sh) break;
    const int key = find_key(ws.tile_off, ws.n_keys, item);
    const int j = key % P.max_chunks;
    const int bg = key / P.max_chunks;
    const int g = bg % P.Hkv, b = bg / P.Hkv;
    const int p0 = ws.offsets[key] + (item - ws.tile_off[key]) * kItemPairs;
    const int p1 = min(p0 + kItemPairs, ws.offsets[key + 1]);
    const int n_tiles = (p1 - p0 + kRows - 1) / kRows;

    // K and V of this chunk (only when the chunk changes)
    if (key != prev_key) {
      const int64_t page = page_of(P, b, j);
      const uint16_t* kp = reinterpret_cast<const uint16_t*>(P.pages) +
                           (page >= 0 ? page_offset(P, page, 0, g, 0) : 0);
      const uint16_t* vp = reinterpret_cast<const uint16_t*>(P.pages) +
                           (page >= 0 ? page_offset(P, page, 1, g, 0) : 0);
      const uint32_t bytes = page >= 0 ? 16u : 0u;
      for (int x = tid; x < kChunk * (D / 8); x += kThreads) {
        const int s = x / (D / 8), c = x % (D / 8);
        const uint32_t off = (uint32_t)(c >> 3) * (kChunk * 128) + tc::swz(s, c & 7);
        tc::cp_async16(sbase + Lay::kK + off, kp + s * D + c * 8, bytes);
        tc::cp_async16(sbase + Lay::kV + off, vp + s * D + c * 8, bytes);
      }
      prev_key = key;
    }
    // first tile's query rows (pair id and weight of this thread's row are
    // fetched one tile ahead, so no dependent global load sits on the tile's path)
    int buf = 0;
    int32_t pid = p0 + tid < p1 ? ws.pairs[p0 + tid] : -1;
    gather_q_row<D>(P, sbase + Lay::kQ0, tid, pid);
    tc::cp_async_commit();
    float w_next = pid >= 0 ? ws.w[pid] : 0.f;

    for (int t = 0; t < n_tiles; ++t) {
      const uint32_t q_cur = sbase + (buf ? Lay::kQ1 : Lay::kQ0);
      const uint32_t q_nxt = sbase + (buf ? Lay::kQ0 : Lay::kQ1);
      tc::cp_async_wait<0>();
      tc::fence_proxy_async();
      tc::tc_fence_before();
      __syncthreads();
      // S = Q K^T
      if (tid == 0) {
        tc::tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t a = tc::smem_desc(q_cur + (kk >> 2) * (kRows * 128) + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = tc::smem_desc(sbase + Lay::kK + (kk >> 2) * (kChunk * 128) + (kk & 3) * 32, 16, 1024);
          tc::mma_bf16(tmem_s, a, bd, kIdS, kk > 0);
        }
        tc::mma_commit(&bar_s);
      }
      // this thread's pair for the current tile
      const int32_t my_pid = pid;
      const float wj = w_next;
      int nk = kChunk;
      if (my_pid >= 0) {
        const int64_t r = my_pid / P.k;
        const int64_t pos = P.pos0 + (r / P.Hq) % P.L;
        if (pos / kChunk == j) nk = (int)(pos - (int64_t)j * kChunk + 1);
      }
      pid_sh[tid] = my_pid;
      // prefetch the next tile's query rows into the other buffer
      if (t + 1 < n_tiles) {
        const int pn = p0 + (t + 1) * kRows + tid;
        pid = pn < p1 ? ws.pairs[pn] : -1;
        gather_q_row<D>(P, q_nxt, tid, pid);
        tc::cp_async_commit();
        w_next = pid >= 0 ? ws.w[pid] : 0.f;
      }
      if (!tc::mbar_wait(&bar_s, phase_s)) abort_sh = 1;
      phase_s ^= 1;
      tc::tc_fence_after();
      // softmax of this thread's row (TMEM lane tid), P -> bf16 over the Q tile
      uint32_t sr[64];
      {
        uint32_t a[32], c[32];
        tc::tmem_ld32(tmem_s + lane_off, a);
        tc::tmem_ld32(tmem_s + lane_off + 32, c);
        tc::tmem_ld_wait();
#pragma unroll
        for (int x = 0; x < 32; ++x) {
          sr[x] = a[x];
          sr[32 + x] = c[x];
        }
      }
      float m = -INFINITY;
#pragma unroll
      for (int x = 0; x < 64; ++x)
        if (x < nk) m = fmaxf(m, __uint_as_float(sr[x]));
      float l = 0.f;
      uint32_t pk[32];
#pragma unroll
      for (int x = 0; x < 64; x += 2) {
        const float e0 = x < nk ? exp2f((__uint_as_float(sr[x]) - m) * scale_log2) : 0.f;
        const float e1 = x + 1 < nk ? exp2f((__uint_as_float(sr[x + 1]) - m) * scale_log2) : 0.f;
        const uint32_t pp = tc::pack_bf16x2(e0, e1);
        pk[x >> 1] = pp;
        l += __uint_as_float(pp << 16) + __uint_as_float(pp & 0xFFFF0000u);
      }
      uint8_t* prow = smem + (q_cur - sbase);
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        uint4 v = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        *reinterpret_cast<uint4*>(prow + tc::swz(tid, c)) = v;
      }
      tc::fence_proxy_async();
      tc::tc_fence_before();
      __syncthreads();
      // O = P V
      if (tid == 0) {
        tc::tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kChunk / 16; ++kk) {
          const uint64_t a = tc::smem_desc(q_cur + kk * 32, 16, 1024);
          const uint64_t bd = tc::smem_desc(sbase + Lay::kV + kk * 2048, kChunk * 128, 1024);
          tc::mma_bf16(tmem_o, a, bd, kIdO, kk > 0);
        }
        tc::mma_commit(&bar_o);
      }
      if (!tc::mbar_wait(&bar_o, phase_o)) abort_sh = 1;
      phase_o ^= 1;
      tc::tc_fence_after();
      // epilogue: O * (w / l) -> bf16 row staged over the P/Q tile (16-byte chunk c
      // of row r at chunk slot c ^ (r & 7): conflict-free), then coalesced stores
      const float sc = (my_pid >= 0 && l > 0.f) ? wj / l : 0.f;
      uint8_t* orow = smem + (q_cur - sbase) + tid * (D * 2);
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t o[32];
        tc::tmem_ld32(tmem_o + lane_off + c0, o);
        tc::tmem_ld_wait();
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          uint32_t w4[4];
#pragma unroll
          for (int u = 0; u < 4; ++u)
            w4[u] = tc::pack_bf16x2(__uint_as_float(o[q4 * 8 + 2 * u]) * sc,
                                    __uint_as_float(o[q4 * 8 + 2 * u + 1]) * sc);
          const int c = (c0 >> 3) + q4;
          *reinterpret_cast<uint4*>(orow + ((c ^ (tid & 7)) << 4)) =
              make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
      }
      // the staged rows are written by whole warps: lane x stores 4-byte word x (+32...)
      __syncthreads();
      {
        const int tile_base = p0 + t * kRows;
        const uint32_t* stg = reinterpret_cast<const uint32_t*>(smem + (q_cur - sbase));
        for (int rr = warp; rr < kRows; rr += kThreads / 32) {
          const int pi = tile_base + rr;
          if (pi >= p1) break;
          const int32_t rp = pid_sh[rr];
          uint32_t* dst = reinterpret_cast<uint32_t*>(ws.partial) + (int64_t)rp * (D / 2);
#pragma unroll
          for (int x = tid & 31; x < D / 2; x += 32)
            dst[x] = stg[rr * (D / 2) + ((((x >> 2) ^ (rr & 7)) << 2) | (x & 3))];
        }
      }
      buf ^= 1;
    }
  }
  if (abort_sh && tid == 0) set_device_error(kErrTimeout);
  tc::cp_async_wait<0>();
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, kTmemCols);
}

// out[row] = sum over valid slots of partial[row * k + slot]  (float32, slot order)
template <int D>
__global__ void merge_kernel(Params P, PrefillWs ws, const int32_t* idx, void* out, int64_t rows) {
  const int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  constexpr int E = D / 32;  // elements per lane
  float acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
  for (int s = 0; s < P.k; ++s) {
    if (idx[r * P.k + s] < 0) continue;
    const uint16_t* src = reinterpret_cast<const uint16_t*>(ws.partial) + (r * P.k + s) * D + lane * E;
    if (E == 4) {
      const uint2 v = *reinterpret_cast<const uint2*>(src);
      acc[0] += __uint_as_float(v.x << 16);
      acc[1] += __uint_as_float(v.x & 0xFFFF0000u);
      acc[2] += __uint_as_float(v.y << 16);
      acc[3] += __uint_as_float(v.y & 0xFFFF0000u);
    } else {
      const uint32_t v = *reinterpret_cast<const uint32_t*>(src);
      acc[0] += __uint_as_float(v << 16);
      acc[1] += __uint_as_float(v & 0xFFFF0000u);
    }
  }
  uint16_t* o = reinterpret_cast<uint16_t*>(out) + r * D + lane * E;
  if (E == 4) {
    *reinterpret_cast<uint2*>(o) = make_uint2(tc::pack_bf16x2(acc[0], acc[1]),
                                              tc::pack_bf16x2(acc[2], acc[3]));
  } else {
    *reinterpret_cast<uint32_t*>(o) = tc::pack_bf16x2(acc[0], acc[1]);
  }
}

template <int D>
cudaError_t run_attn_tc(const Params& P, void* out, const int32_t* idx, const PrefillWs& ws,
                        cudaStream_t s) {
  using Lay = AttnLayout<D>;
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)Lay::kSmem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if ((e = cudaMemsetAsync(ws.queue, 0, sizeof(int32_t), s)) != cudaSuccess) return e;
  {
    HILS_PROFILE("prefill.attend_tc", s);
    attn_tc_kernel<D><<<2 * sms, kThreads, Lay::kSmem, s>>>(P, ws);
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int64_t rows = (int64_t)P.B * P.L * P.Hq;
  {
    HILS_PROFILE("prefill.merge", s);
    merge_kernel<D><<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(P, ws, idx, out, rows);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_tc(const Params& P, void* out, const int32_t* idx, const PrefillWs& ws,
                           cudaStream_t s) {
  return P.d == 64 ? run_attn_tc<64>(P, out, idx, ws, s) : run_attn_tc<128>(P, out, idx, ws, s);
}

}  // namespace hils
