// Prefill forward on CUDA cores: a1..a7 without materialising scores.
//
//   select   one thread per query row: q~ in registers, landmark tiles of the
//            row's KV head staged in shared memory, a running sorted list of
//            the k-1 best candidates (strict '>' while chunks are visited in
//            ascending order keeps the lower index on ties), then the fusion
//            softmax over own + selected.
//   bucket   counting sort of the (row, slot) pairs by (sequence, KV head,
//            chunk), so that every chunk's K/V tile is read once per tile of
//            up to kTilePairs rows that selected it (key-major grouping).
//   attend   per tile: K/V of the chunk in shared memory, one warp per pair:
//            scores, masked softmax (own chunk causal), P.V, and the
//            w/l-scaled result added into a float32 accumulator row.
//   finish   accumulator -> output dtype.
#include <cfloat>

#include "hils_common.cuh"

namespace hils {
namespace {

constexpr int kSelThreads = 128;
constexpr int kLmTile = 32;
constexpr int kTilePairs = 128;
constexpr int kAttThreads = 256;
constexpr int kAttWarps = kAttThreads / 32;
constexpr int kBucketWindow = 8192;   // query positions per bucketing window
constexpr int kBucketRows = 256;      // query positions per bucketing CTA
constexpr int kHistMax = 24576;       // chunk bins a bucketing CTA keeps in shared memory
constexpr int64_t kMaxKeys = 1 << 26; // bucket keys above which windows are dropped

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

template <int D>
__global__ void __launch_bounds__(kSelThreads) select_kernel(Params P, int32_t* idx, float* w) {
  extern __shared__ float smem[];
  const int t = threadIdx.x;
  const int h = blockIdx.y, b = blockIdx.z;
  const int g = h / P.group;
  const int64_t i = (int64_t)blockIdx.x * kSelThreads + t;
  const bool valid = i < P.L;
  const int64_t pos = P.pos0 + (valid ? i : P.L - 1);
  const int64_t own = pos / kChunk;
  const int64_t r = ((int64_t)b * P.L + i) * P.Hq + h;
  const int64_t i_last = min((int64_t)(blockIdx.x + 1) * kSelThreads, P.L) - 1;
  const int64_t own_max = (P.pos0 + i_last) / kChunk;

  float qt[D];
#pragma unroll
  for (int e = 0; e < D; e += 8) {
    if (valid) {
      load8(P.q, P.dtype, r * D + e, &qt[e]);
    } else {
#pragma unroll
      for (int u = 0; u < 8; ++u) qt[e + u] = 0.f;
    }
  }

  // a1: calibration, with A and B staged in shared memory (phase 1 layout)
  if (P.r > 0) {
    float* sA = smem;
    float* sB = sA + D * P.r;
    float* sT = sB + P.r * D;
    for (int x = t; x < D * P.r; x += kSelThreads) {
      sA[x] = P.A[x];
      sB[x] = P.Bm[x];
    }
    __syncthreads();
    for (int a = 0; a < P.r; ++a) {
      float acc = 0.f;
#pragma unroll
      for (int e = 0; e < D; ++e) acc = fmaf(qt[e], sA[e * P.r + a], acc);
      sT[a * kSelThreads + t] = acc;
    }
    for (int a = 0; a < P.r; ++a) {
      const float ta = sT[a * kSelThreads + t];
#pragma unroll
      for (int e = 0; e < D; ++e) qt[e] = fmaf(ta, sB[a * D + e], qt[e]);
    }
    __syncthreads();
  }

  // a2 + a3: stream the landmarks, keep the best k-1 candidates (phase 2 layout)
  const int K = P.k - 1;
  float* sLm = smem;
  float* lsS = sLm + kLmTile * D;
  int* lsJ = reinterpret_cast<int*>(lsS + kMaxTopK * kSelThreads);
  int n = 0;
  float thr = -INFINITY;
  float s_own = 0.f;
  for (int64_t j0 = 0; j0 <= own_max; j0 += kLmTile) {
    __syncthreads();
    for (int x = t; x < kLmTile * (D / 8); x += kSelThreads) {
      const int jj = x / (D / 8), e8 = (x % (D / 8)) * 8;
      const int64_t j = j0 + jj;
      if (j <= own_max) {
        load8(P.landmarks, P.dtype, (((int64_t)b * P.max_chunks + j) * P.Hkv + g) * D + e8,
              &sLm[jj * D + e8]);
      }
    }
    __syncthreads();
    for (int jj = 0; jj < kLmTile; ++jj) {
      const int64_t j = j0 + jj;
      if (j > own) break;
      float acc = 0.f;
#pragma unroll
      for (int e = 0; e < D; ++e) acc = fmaf(qt[e], sLm[jj * D + e], acc);
      const float s = acc * P.inv_sqrt_d;
      if (j == own) {
        s_own = s;
      } else if (K > 0 && (n < K || s > thr)) {
        int p = n < K ? n : K - 1;
        while (p > 0 && s > lsS[(p - 1) * kSelThreads + t]) {
          lsS[p * kSelThreads + t] = lsS[(p - 1) * kSelThreads + t];
          lsJ[p * kSelThreads + t] = lsJ[(p - 1) * kSelThreads + t];
          --p;
        }
        lsS[p * kSelThreads + t] = s;
        lsJ[p * kSelThreads + t] = (int)j;
        if (n < K) ++n;
        if (n == K) thr = lsS[(K - 1) * kSelThreads + t];
      }
    }
  }
  if (!valid) return;

  // a4: fusion weights
  float m = s_own;
  for (int a = 0; a < n; ++a) m = fmaxf(m, lsS[a * kSelThreads + t]);
  float z = __expf(s_own - m);
  for (int a = 0; a < n; ++a) z += __expf(lsS[a * kSelThreads + t] - m);
  const float iz = 1.f / z;
  int32_t* ix = idx + r * P.k;
  float* wr = w + r * P.k;
  ix[0] = (int32_t)own;
  wr[0] = __expf(s_own - m) * iz;
  for (int a = 0; a < n; ++a) {
    ix[1 + a] = lsJ[a * kSelThreads + t];
    wr[1 + a] = __expf(lsS[a * kSelThreads + t] - m) * iz;
  }
  for (int a = n + 1; a < P.k; ++a) {
    ix[a] = -1;
    wr[a] = 0.f;
  }
}

// ---- bucketing ------------------------------------------------------------
// Keys are (sequence, KV head, query window, chunk): the attention kernels take
// work items in key order, so the items running at the same time read the
// query rows of one window of kBucketWindow positions, which stay in L2.
struct Windows {
  int n;            // windows per sequence
  int64_t rows;     // query positions per window (a multiple of kBucketRows)
};

__device__ __forceinline__ int64_t bucket_key(const Params& P, Windows W, int b, int g, int64_t i,
                                              int32_t j) {
  return (((int64_t)b * P.Hkv + g) * W.n + i / W.rows) * P.max_chunks + j;
}

// Pair p = row * k + slot of row (b, i, h) -> its key (global-atomic fallback path).
__device__ __forceinline__ int64_t pair_key(const Params& P, Windows W, int64_t p, int32_t j) {
  const int64_t r = p / P.k;
  const int h = (int)(r % P.Hq);
  const int64_t bi = r / P.Hq;
  return bucket_key(P, W, (int)(bi / P.L), h / P.group, bi % P.L, j);
}

// The 8-byte record of pair (query row, chunk j) for the tensor-core
// attention: the row, and the fusion weight w with its 6 lowest mantissa bits
// replaced by the number of keys of chunk j visible to the row, minus one.
// The visible keys are 64 except in the row's own chunk, where they end at
// the row's position.  The change to w, below 2^-17 of w, is far below the
// bf16 rounding of the probabilities that w scales.
__device__ __forceinline__ int2 pair_record(int32_t row, float w, int64_t pos, int32_t j) {
  const int nk = pos / kChunk == j ? (int)(pos - (int64_t)j * kChunk + 1) : kChunk;
  return make_int2(row, (int)((__float_as_uint(w) & ~63u) | (uint32_t)(nk - 1)));
}

// One CTA per (sequence b, KV head g, block of kBucketRows query positions):
// the block's pairs are counted into a shared-memory histogram over the chunks
// its rows can see, then added to the global counts once per nonzero bin.
// Every pair of a position i of the group's heads is one run of group * k
// consecutive idx entries.
// x / d for small x (x, d < 2^16) by a multiply-high with m = 2^32 / d rounded
// up; d = 1 (where m would not fit) returns x.
struct SmallDiv {
  uint32_t d, m;
  __device__ __forceinline__ explicit SmallDiv(uint32_t dd)
      : d(dd), m(dd > 1 ? 0xFFFFFFFFu / dd + 1u : 0u) {}
  __device__ __forceinline__ uint32_t div(uint32_t x) const { return d > 1 ? __umulhi(x, m) : x; }
};

// Pairs a thread takes per round of the bucketing loops: their loads are all
// issued before the first is used.
constexpr int kBucketUnroll = 8;

__device__ __forceinline__ void block_hist(const Params& P, const int32_t* idx, int32_t* hist,
                                           int nvis, int64_t i0, int64_t i1, int b, int g,
                                           bool check) {
  const int per_i = P.group * P.k;
  const SmallDiv dv(per_i);
  const int n = (int)(i1 - i0) * per_i;
  const int32_t* base = idx + (((int64_t)b * P.L + i0) * P.Hq + g * P.group) * P.k;
  const int64_t row_stride = (int64_t)P.Hq * P.k;   // idx entries from one position to the next
  for (int f0 = threadIdx.x; f0 < n; f0 += blockDim.x * kBucketUnroll) {
    int32_t j[kBucketUnroll];
#pragma unroll
    for (int u = 0; u < kBucketUnroll; ++u) {
      const int f = f0 + u * blockDim.x;
      const int ii = (int)dv.div((uint32_t)f);
      j[u] = f < n ? __ldg(base + ii * row_stride + (f - ii * per_i)) : -1;
    }
#pragma unroll
    for (int u = 0; u < kBucketUnroll; ++u) {
      if (j[u] < 0) continue;
      if (j[u] >= nvis) {
        if (check) set_device_error(kErrChunk);
        continue;
      }
      atomicAdd(&hist[j[u]], 1);
    }
  }
}

__global__ void __launch_bounds__(256) bucket_count_kernel(Params P, const int32_t* idx,
                                                           int32_t* counts, Windows W) {
  extern __shared__ int32_t hist[];
  const int b = blockIdx.z, g = blockIdx.y;
  const int64_t i0 = (int64_t)blockIdx.x * kBucketRows, i1 = min(i0 + kBucketRows, P.L);
  const int nvis = (int)min((int64_t)P.max_chunks, (P.pos0 + i1 - 1) / kChunk + 1);
  for (int x = threadIdx.x; x < nvis; x += blockDim.x) hist[x] = 0;
  __syncthreads();
  block_hist(P, idx, hist, nvis, i0, i1, b, g, true);
  __syncthreads();
  const int64_t kb = bucket_key(P, W, b, g, i0, 0);
  for (int x = threadIdx.x; x < nvis; x += blockDim.x)
    if (hist[x]) atomicAdd(&counts[kb + x], hist[x]);
}

// Same blocks: one global atomic per nonzero bin reserves the block's range of
// each bucket, shared-memory atomics place the pairs inside it.
__global__ void __launch_bounds__(256, 3) bucket_scatter_kernel(Params P, const int32_t* idx,
                                                             const float* wts, int32_t* cursor,
                                                             int32_t* pairs, int2* pinfo,
                                                             Windows W) {
  extern __shared__ int32_t hist[];
  const int b = blockIdx.z, g = blockIdx.y;
  const int64_t i0 = (int64_t)blockIdx.x * kBucketRows, i1 = min(i0 + kBucketRows, P.L);
  const int nvis = (int)min((int64_t)P.max_chunks, (P.pos0 + i1 - 1) / kChunk + 1);
  int32_t* base = hist + nvis;
  for (int x = threadIdx.x; x < nvis; x += blockDim.x) hist[x] = 0;
  __syncthreads();
  block_hist(P, idx, hist, nvis, i0, i1, b, g, false);
  __syncthreads();
  const int64_t kb = bucket_key(P, W, b, g, i0, 0);
  for (int x = threadIdx.x; x < nvis; x += blockDim.x) {
    const int32_t c = hist[x];
    base[x] = c ? atomicAdd(&cursor[kb + x], c) : 0;
    hist[x] = 0;
  }
  __syncthreads();
  const int per_i = P.group * P.k;
  const SmallDiv dv(per_i), dk(P.k);
  const int n = (int)(i1 - i0) * per_i;
  const bool rows_out = pinfo != nullptr;   // tensor-core path: a record per pair
  for (int f0 = threadIdx.x; f0 < n; f0 += blockDim.x * kBucketUnroll) {
    int32_t j[kBucketUnroll];
    float wv[kBucketUnroll];
#pragma unroll
    for (int u = 0; u < kBucketUnroll; ++u) {
      const int f = f0 + u * blockDim.x;
      const int ii = (int)dv.div((uint32_t)f);
      const int64_t p = (((int64_t)b * P.L + i0 + ii) * P.Hq + g * P.group) * P.k + (f - ii * per_i);
      j[u] = f < n ? __ldg(idx + p) : -1;
      wv[u] = (f < n && rows_out) ? __ldg(wts + p) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < kBucketUnroll; ++u) {
      if (j[u] < 0 || j[u] >= nvis) continue;
      const int f = f0 + u * blockDim.x;
      const int ii = (int)dv.div((uint32_t)f);
      const int q = f - ii * per_i;                                        // head-in-group * k + slot
      const int64_t i = i0 + ii;
      const int64_t row0 = ((int64_t)b * P.L + i) * P.Hq + g * P.group;   // first row of the group
      const int32_t at = base[j[u]] + atomicAdd(&hist[j[u]], 1);
      if (rows_out)
        pinfo[at] = pair_record((int32_t)(row0 + dk.div((uint32_t)q)), wv[u], P.pos0 + i, j[u]);
      else
        pairs[at] = (int32_t)(row0 * P.k + q);
    }
  }
}

// Fallback when a block's visible chunks do not fit in shared memory.
__global__ void count_kernel(Params P, const int32_t* idx, int32_t* counts, int64_t n_pairs,
                             Windows W) {
  const int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (p >= n_pairs) return;
  const int32_t j = idx[p];
  if (j < 0) return;
  if (j >= P.max_chunks) {
    set_device_error(kErrChunk);
    return;
  }
  atomicAdd(&counts[pair_key(P, W, p, j)], 1);
}

__global__ void scatter_kernel(Params P, const int32_t* idx, const float* wts, int32_t* cursor,
                               int32_t* pairs, int2* pinfo, int64_t n_pairs, Windows W) {
  const int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (p >= n_pairs) return;
  const int32_t j = idx[p];
  if (j < 0 || j >= P.max_chunks) return;
  const int32_t at = atomicAdd(&cursor[pair_key(P, W, p, j)], 1);
  if (pinfo) {
    const int64_t r = p / P.k;
    pinfo[at] = pair_record((int32_t)r, wts[p], P.pos0 + (r / P.Hq) % P.L, j);
  } else {
    pairs[at] = (int32_t)p;
  }
}

// Exclusive scans of the bucket sizes (pair offsets) and of their work items
// (ceil(count / tile_pairs) each), and (key, first pair, end pair) of every
// work item: two passes over blocks of kScanBlock keys.  Pass 1 writes every
// block's pair and item totals; pass 2 gives each block its prefix (the sum
// of the earlier blocks' totals) and scans inside the block.
constexpr int kScanBlock = 1024;

__device__ __forceinline__ int2 block_sum_pairs_items(int2 v, int2* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    v.x += __shfl_xor_sync(0xffffffffu, v.x, o);
    v.y += __shfl_xor_sync(0xffffffffu, v.y, o);
  }
  if (lane == 0) red[warp] = v;
  __syncthreads();
  int2 t = make_int2(0, 0);
  if (threadIdx.x < 32) {
    t = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : make_int2(0, 0);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      t.x += __shfl_xor_sync(0xffffffffu, t.x, o);
      t.y += __shfl_xor_sync(0xffffffffu, t.y, o);
    }
  }
  return t;   // valid in warp 0
}

__global__ void __launch_bounds__(kScanBlock) scan_totals_kernel(const int32_t* counts, int n_keys,
                                                                 int tile_pairs, int2* totals) {
  __shared__ int2 red[32];
  const int key = blockIdx.x * kScanBlock + threadIdx.x;
  const int c = key < n_keys ? counts[key] : 0;
  const int2 t = block_sum_pairs_items(make_int2(c, (c + tile_pairs - 1) / tile_pairs), red);
  if (threadIdx.x == 0) totals[blockIdx.x] = t;
}

__global__ void __launch_bounds__(kScanBlock) scan_kernel(const int32_t* counts, int n_keys,
                                                          int tile_pairs, const int2* totals,
                                                          int32_t* offsets, int32_t* tile_off,
                                                          int32_t* cursor, int4* items) {
  __shared__ int2 red[32];
  __shared__ int2 base_sh;
  __shared__ int2 wsum[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // prefix of this block: the totals of the blocks before it
  int2 pre = make_int2(0, 0);
  for (int x = tid; x < (int)blockIdx.x; x += kScanBlock) {
    const int2 t = totals[x];
    pre.x += t.x;
    pre.y += t.y;
  }
  const int2 bt = block_sum_pairs_items(pre, red);
  if (tid == 0) base_sh = bt;
  // inclusive scan of (pairs, items) inside the block
  const int key = blockIdx.x * kScanBlock + tid;
  const int c = key < n_keys ? counts[key] : 0;
  const int nt = (c + tile_pairs - 1) / tile_pairs;
  int2 v = make_int2(c, nt);
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int ax = __shfl_up_sync(0xffffffffu, v.x, o), ay = __shfl_up_sync(0xffffffffu, v.y, o);
    if (lane >= o) {
      v.x += ax;
      v.y += ay;
    }
  }
  if (lane == 31) wsum[warp] = v;
  __syncthreads();
  if (warp == 0) {
    int2 w = lane < (kScanBlock >> 5) ? wsum[lane] : make_int2(0, 0);
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int ax = __shfl_up_sync(0xffffffffu, w.x, o), ay = __shfl_up_sync(0xffffffffu, w.y, o);
      if (lane >= o) {
        w.x += ax;
        w.y += ay;
      }
    }
    wsum[lane] = w;   // inclusive over warps
  }
  __syncthreads();
  const int2 wp = warp > 0 ? wsum[warp - 1] : make_int2(0, 0);
  const int po = base_sh.x + wp.x + v.x - c;    // exclusive pair offset
  const int to = base_sh.y + wp.y + v.y - nt;   // exclusive item offset
  if (key < n_keys) {
    offsets[key] = po;
    cursor[key] = po;
    tile_off[key] = to;
    for (int u = 0; u < nt; ++u)
      items[to + u] = make_int4(key, po + u * tile_pairs, min(po + (u + 1) * tile_pairs, po + c), 0);
    if (key == n_keys - 1) {
      offsets[n_keys] = po + c;
      tile_off[n_keys] = to + nt;
    }
  }
}

// ---- attention over key-major tiles ------------------------------------
template <int D>
__global__ void __launch_bounds__(kAttThreads) attend_kernel(Params P, PrefillWs ws) {
  extern __shared__ float sm[];
  constexpr int LD = D + 1;  // padded row stride: conflict-free column reads
  float* sK = sm;
  float* sV = sK + kChunk * LD;
  float* sQ = sV + kChunk * LD;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tile = blockIdx.x;
  if (tile >= ws.tile_off[ws.n_keys]) return;
  const int4 item = ws.items[tile];
  const int key = item.x;
  const int j = key % P.max_chunks;
  const int bg = key / P.max_chunks / ws.n_win;
  const int g = bg % P.Hkv, b = bg / P.Hkv;
  const int64_t page = page_of(P, b, j);
  if (page < 0) return;
  for (int x = tid; x < kChunk * (D / 8); x += kAttThreads) {
    const int s = x / (D / 8), e8 = (x % (D / 8)) * 8;
    float v[8];
    load8(P.pages, P.dtype, page_offset(P, page, 0, g, s) + e8, v);
#pragma unroll
    for (int u = 0; u < 8; ++u) sK[s * LD + e8 + u] = v[u];
    load8(P.pages, P.dtype, page_offset(P, page, 1, g, s) + e8, v);
#pragma unroll
    for (int u = 0; u < 8; ++u) sV[s * LD + e8 + u] = v[u];
  }
  __syncthreads();
  const int p0 = item.y, p1 = item.z;
  float* q = sQ + warp * D;
  for (int p = p0 + warp; p < p1; p += kAttWarps) {
    const int32_t pid = ws.pairs[p];
    const int64_t r = pid / P.k;
    const int64_t i = (r / P.Hq) % P.L;
    const int64_t pos = P.pos0 + i;
    const int nk = (pos / kChunk == j) ? (int)(pos - (int64_t)j * kChunk + 1) : kChunk;
    if (lane < D / 8) load8(P.q, P.dtype, r * D + lane * 8, &q[lane * 8]);
    __syncwarp();
    float s0 = 0.f, s1 = 0.f;
#pragma unroll 8
    for (int e = 0; e < D; ++e) {
      s0 = fmaf(q[e], sK[lane * LD + e], s0);
      s1 = fmaf(q[e], sK[(lane + 32) * LD + e], s1);
    }
    s0 = lane < nk ? s0 * P.inv_sqrt_d : -INFINITY;
    s1 = lane + 32 < nk ? s1 * P.inv_sqrt_d : -INFINITY;
    const float m = warp_max(fmaxf(s0, s1));
    const float e0 = __expf(s0 - m), e1 = __expf(s1 - m);
    const float l = warp_sum(e0 + e1);
    float o[D / 32];
#pragma unroll
    for (int a = 0; a < D / 32; ++a) o[a] = 0.f;
    for (int kk = 0; kk < kChunk; ++kk) {
      const float pk = __shfl_sync(0xffffffffu, kk < 32 ? e0 : e1, kk & 31);
#pragma unroll
      for (int a = 0; a < D / 32; ++a) o[a] = fmaf(pk, sV[kk * LD + lane + 32 * a], o[a]);
    }
    const float scale = ws.w[pid] / l;
    float* acc = ws.acc + r * D;
#pragma unroll
    for (int a = 0; a < D / 32; ++a) atomicAdd(&acc[lane + 32 * a], o[a] * scale);
    __syncwarp();
  }
}

__global__ void finish_kernel(Params P, const float* acc, void* out, int64_t n) {
  const int64_t x = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (x < n) store_elem(out, P.dtype, x, acc[x]);
}

template <int D>
size_t select_smem(int r) {
  const size_t ph1 = (size_t)(2 * D * r + r * kSelThreads) * sizeof(float);
  const size_t ph2 = (size_t)(kLmTile * D + 2 * kMaxTopK * kSelThreads) * sizeof(float);
  return ph1 > ph2 ? ph1 : ph2;
}

template <int D>
constexpr size_t attend_smem() {
  return (size_t)(2 * kChunk * (D + 1) + kAttWarps * D) * sizeof(float);
}

template <int D>
cudaError_t run_prefill(const Params& P, void* out, const PrefillWs& ws, cudaStream_t s) {
  const int64_t rows = (int64_t)P.B * P.L * P.Hq;
  const int64_t n_pairs = rows * P.k;
  cudaError_t e;
  // a1..a4
  if (P.dtype == HILS_BF16) {
    if ((e = launch_select_tc(P, ws, ws.idx, ws.w, s)) != cudaSuccess) return e;
  } else {
    const size_t ssm = select_smem<D>(P.r);
    e = set_smem(select_kernel<D>, ssm);
    if (e != cudaSuccess) return e;
    dim3 sg((unsigned)((P.L + kSelThreads - 1) / kSelThreads), P.Hq, P.B);
    {
      HILS_PROFILE("prefill.select", s);
      select_kernel<D><<<sg, kSelThreads, ssm, s>>>(P, ws.idx, ws.w);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  // bucket by (sequence, KV head, chunk)
  e = launch_bucketing(P, ws.idx, ws.w, ws, P.dtype == HILS_BF16,
                       P.dtype == HILS_BF16 ? kItemPairs : kTilePairs, "prefill.bucket", s);
  if (e != cudaSuccess) return e;
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // a5 + a6
  if (P.dtype == HILS_BF16) return launch_attn_tc(P, out, ws, s);
  if ((e = cudaMemsetAsync(ws.acc, 0, sizeof(float) * rows * D, s)) != cudaSuccess) return e;
  constexpr size_t asm_ = attend_smem<D>();
  e = set_smem(attend_kernel<D>, asm_);
  if (e != cudaSuccess) return e;
  {
    HILS_PROFILE("prefill.attend", s);
    attend_kernel<D><<<(unsigned)ws.max_tiles, kAttThreads, asm_, s>>>(P, ws);
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int64_t n = rows * D;
  {
    HILS_PROFILE("prefill.finish", s);
    finish_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(P, ws.acc, out, n);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bucketing(const Params& P, const int32_t* idx, const float* wts,
                             const PrefillWs& ws, bool records, int tile_pairs, const char* label,
                             cudaStream_t s) {
  const int64_t n_pairs = (int64_t)P.B * P.L * P.Hq * P.k;
  cudaError_t e;
  if ((e = cudaMemsetAsync(ws.counts, 0, sizeof(int32_t) * ws.n_keys, s)) != cudaSuccess) return e;
  HILS_PROFILE(label, s);
  const Windows W{ws.n_win, ws.win_rows};
  const int64_t nvis_max = min((int64_t)P.max_chunks, (P.pos0 + P.L - 1) / kChunk + 1);
  const size_t hsm = sizeof(int32_t) * 2 * (size_t)nvis_max;
  const unsigned nb = (unsigned)((ws.n_keys + kScanBlock - 1) / kScanBlock);
  int2* rec = records ? ws.pinfo : nullptr;
  if (nvis_max <= kHistMax) {
    if ((e = set_smem(bucket_scatter_kernel, hsm)) != cudaSuccess) return e;
    if ((e = set_smem(bucket_count_kernel, hsm)) != cudaSuccess) return e;
    const dim3 bgrid((unsigned)((P.L + kBucketRows - 1) / kBucketRows), P.Hkv, P.B);
    bucket_count_kernel<<<bgrid, 256, hsm / 2, s>>>(P, idx, ws.counts, W);
    scan_totals_kernel<<<nb, kScanBlock, 0, s>>>(ws.counts, ws.n_keys, tile_pairs, ws.scan_totals);
    scan_kernel<<<nb, kScanBlock, 0, s>>>(ws.counts, ws.n_keys, tile_pairs, ws.scan_totals,
                                          ws.offsets, ws.tile_off, ws.cursor, ws.items);
    bucket_scatter_kernel<<<bgrid, 256, hsm, s>>>(P, idx, wts, ws.cursor, ws.pairs, rec, W);
  } else {
    const unsigned pb = (unsigned)((n_pairs + 255) / 256);
    count_kernel<<<pb, 256, 0, s>>>(P, idx, ws.counts, n_pairs, W);
    scan_totals_kernel<<<nb, kScanBlock, 0, s>>>(ws.counts, ws.n_keys, tile_pairs, ws.scan_totals);
    scan_kernel<<<nb, kScanBlock, 0, s>>>(ws.counts, ws.n_keys, tile_pairs, ws.scan_totals,
                                          ws.offsets, ws.tile_off, ws.cursor, ws.items);
    scatter_kernel<<<pb, 256, 0, s>>>(P, idx, wts, ws.cursor, ws.pairs, rec, n_pairs, W);
  }
  return cudaGetLastError();
}

static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Workspace carve-up; with base == nullptr only the size is computed.
// Query windows of the bucket keys, unless the key space would grow past kMaxKeys.
static void bucket_windows(const Params& P, int* n_win, int64_t* win_rows) {
  *n_win = (int)((P.L + kBucketWindow - 1) / kBucketWindow);
  *win_rows = kBucketWindow;
  if ((int64_t)P.B * P.Hkv * *n_win * P.max_chunks > kMaxKeys) {
    *n_win = 1;
    *win_rows = P.L > 0 ? P.L : 1;
  }
}

size_t prefill_ws_bytes(const Params& P, PrefillWs* ws, char* base) {
  const int64_t rows = (int64_t)P.B * P.L * P.Hq;
  const int64_t n_pairs = rows * P.k;
  int n_win;
  int64_t win_rows;
  bucket_windows(P, &n_win, &win_rows);
  const int64_t n_keys = (int64_t)P.B * P.Hkv * n_win * P.max_chunks;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    char* p = base ? base + off : nullptr;
    off += align256(bytes);
    return p;
  };
  PrefillWs w{};
  w.idx = (int32_t*)take(sizeof(int32_t) * n_pairs);
  w.w = (float*)take(sizeof(float) * n_pairs);
  w.counts = (int32_t*)take(sizeof(int32_t) * n_keys);
  w.offsets = (int32_t*)take(sizeof(int32_t) * (n_keys + 1));
  w.tile_off = (int32_t*)take(sizeof(int32_t) * (n_keys + 1));
  w.cursor = (int32_t*)take(sizeof(int32_t) * n_keys);
  if (P.dtype == HILS_BF16)
    w.pinfo = (int2*)take(sizeof(int2) * n_pairs + 16);   // + 16: tiles are copied in 16-byte units
  else
    w.pairs = (int32_t*)take(sizeof(int32_t) * n_pairs);
  if (P.dtype == HILS_BF16) {
    const int64_t T = (P.L + kScoreTileRows - 1) / kScoreTileRows;
    w.qimg = take((size_t)P.B * P.Hq * T * 3 * kScoreTileRows * P.d * 2);
  } else {
    w.acc = (float*)take(sizeof(float) * rows * P.d);
  }
  w.n_keys = (int)n_keys;
  w.n_win = n_win;
  w.win_rows = win_rows;
  w.max_tiles = (n_pairs + kTilePairs - 1) / kTilePairs + n_keys;
  w.items = (int4*)take(sizeof(int4) * w.max_tiles);
  w.scan_totals = (int2*)take(sizeof(int2) * ((n_keys + 1023) / 1024));
  if (ws) *ws = w;
  return off;
}

size_t backward_ws_bytes(const Params& P, BackwardWs* ws, char* base) {
  const int64_t rows = (int64_t)P.B * P.L * P.Hq;
  const int64_t n_pairs = rows * P.k;
  int n_win;
  int64_t win_rows;
  bucket_windows(P, &n_win, &win_rows);
  const int64_t n_keys = (int64_t)P.B * P.Hkv * n_win * P.max_chunks;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    char* p = base ? base + off : nullptr;
    off += align256(bytes);
    return p;
  };
  BackwardWs w{};
  PrefillWs& k = w.bk;
  k.counts = (int32_t*)take(sizeof(int32_t) * n_keys);
  k.offsets = (int32_t*)take(sizeof(int32_t) * (n_keys + 1));
  k.tile_off = (int32_t*)take(sizeof(int32_t) * (n_keys + 1));
  k.cursor = (int32_t*)take(sizeof(int32_t) * n_keys);
  k.pairs = (int32_t*)take(sizeof(int32_t) * n_pairs);
  k.n_keys = (int)n_keys;
  k.n_win = n_win;
  k.win_rows = win_rows;
  k.max_tiles = (n_pairs + kBackwardTilePairs - 1) / kBackwardTilePairs + n_keys;
  k.items = (int4*)take(sizeof(int4) * k.max_tiles);
  k.scan_totals = (int2*)take(sizeof(int2) * ((n_keys + 1023) / 1024));
  if (backward_on_tc(P)) {
    w.delta = (float*)take(sizeof(float) * rows);
    w.lmc = (float*)take(sizeof(float) * (size_t)P.B * P.max_chunks * P.Hkv * P.d);
    w.vchunk = (float*)take(sizeof(float) * (size_t)P.B * P.max_chunks * P.Hkv * P.d);
    w.mpart = (float*)take(sizeof(float) * (size_t)(kBackwardMaxCtas + 1) * P.d * P.d);
  } else {
    w.dw = (float*)take(sizeof(float) * n_pairs);
  }
  if (ws) *ws = w;
  return off;
}

cudaError_t launch_prefill(const Params& P, void* out, int32_t* idx_out, float* w_out,
                           const PrefillWs& ws_in, cudaStream_t s) {
  PrefillWs ws = ws_in;
  if (idx_out) ws.idx = idx_out;
  if (w_out) ws.w = w_out;
  if (P.L == 0 || P.B == 0) return cudaSuccess;
  return P.d == 64 ? run_prefill<64>(P, out, ws, s) : run_prefill<128>(P, out, ws, s);
}

}  // namespace hils
