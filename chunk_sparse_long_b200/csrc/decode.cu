// Decode step (a8): append, landmark scan + selection, split-k chunk attention.
//
//   scan    grid (n_split, B).  Every CTA computes q~ for all query heads of its
//           sequence, streams the landmarks of its chunk range with 16-byte
//           loads (the per-step cost that grows with context), keeps each
//           head's best k-1 candidates, and takes a ticket per head.  The CTA
//           that takes the last ticket of a head merges that head's lists in
//           (score desc, index asc) order, adds the own chunk and writes the
//           fusion weights.  No CTA waits on another.
//   attend  grid (k, Hq, B): one selected chunk per CTA (64 keys), softmax and
//           P.V, weighted partial result to the workspace; the last CTA of a
//           (sequence, head) sums the k partials in slot order (deterministic).
//
// Selection of the best K among n candidates by one warp ("threshold, then
// select"): tau = the K-th largest of the 32 lane maxima is a lower bound of
// the K-th best candidate (K distinct candidates reach it), so every member
// of the answer has score >= tau.  The survivors (score >= tau) are compacted
// into shared memory and the exact answer is taken there by K rounds of
// "best entry after the previous one" in (score desc, index asc) order.
#include <cfloat>

#include "hils_common.cuh"

namespace hils {
namespace {

constexpr int kScanThreads = 256;
constexpr int kScanWarps = kScanThreads / 32;
constexpr int kMaxSplitChunks = 512;
constexpr int kMergeCap = 512;   // survivors a warp can hold while merging
constexpr unsigned kFull = 0xffffffffu;

__device__ __forceinline__ bool before(float sa, int ja, float sb, int jb) {
  return sa > sb || (sa == sb && ja < jb);
}

// K-th largest of one value per lane (-inf when fewer than K lanes hold one).
__device__ float warp_kth_largest(float v, int K) {
  const int lane = threadIdx.x & 31;
  float m = -INFINITY;
  for (int round = 0; round < K; ++round) {
    m = v;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, o));
    if (m == -INFINITY) return -INFINITY;
    const unsigned holders = __ballot_sync(kFull, v == m);
    if (lane == __ffs(holders) - 1) v = -INFINITY;
  }
  return m;
}

// Exact best-K over n entries in shared memory; result in lane a < K as
// (os, oj), padded with (-inf, -1).  Entries with j < 0 are ignored.
__device__ void warp_select(const float* s, const int* j, int n, int K, float& os, int& oj) {
  const int lane = threadIdx.x & 31;
  os = -INFINITY;
  oj = -1;
  float last_s = INFINITY;
  int last_j = -1;
  for (int slot = 0; slot < K; ++slot) {
    float bs = -INFINITY;
    int bj = INT32_MAX;
    for (int x = lane; x < n; x += 32) {
      const float v = s[x];
      const int vj = j[x];
      if (vj < 0) continue;
      if (before(last_s, last_j, v, vj) && (bj == INT32_MAX || before(v, vj, bs, bj))) {
        bs = v;
        bj = vj;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float xs = __shfl_xor_sync(kFull, bs, o);
      const int xj = __shfl_xor_sync(kFull, bj, o);
      if (xj != INT32_MAX && (bj == INT32_MAX || before(xs, xj, bs, bj))) {
        bs = xs;
        bj = xj;
      }
    }
    if (bj == INT32_MAX) break;
    if (lane == slot) {
      os = bs;
      oj = bj;
    }
    last_s = bs;
    last_j = bj;
  }
}

// Append (s, j) for lanes with keep=true to a warp-private list; returns the new count.
__device__ __forceinline__ int warp_append(bool keep, float s, int j, float* ls, int* lj, int count,
                                           int cap) {
  const int lane = threadIdx.x & 31;
  const unsigned bal = __ballot_sync(kFull, keep);
  const int at = count + __popc(bal & ((1u << lane) - 1u));
  if (keep && at < cap) {
    ls[at] = s;
    lj[at] = j;
  }
  return count + __popc(bal);
}

template <int D>
__global__ void __launch_bounds__(kScanThreads)
    scan_kernel(Params P, const void* k_new, const void* v_new, DecodeWs ws, int32_t* idx_out,
                float* w_out) {
  extern __shared__ float sm[];
  float* sq = sm;                                   // [Hq][D]
  float* sqt = sq + P.Hq * D;                       // [Hq][D]
  float* sT = sqt + P.Hq * D;                       // [Hq][kMaxRank]
  float* sS = sT + P.Hq * kMaxRank;                 // [chunks_per_split][Hq]
  float* wl_s = sS + ws.chunks_per_split * P.Hq;    // [kScanWarps][kMergeCap]
  int* wl_j = reinterpret_cast<int*>(wl_s + kScanWarps * kMergeCap);
  __shared__ unsigned long long last_mask;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, b = blockIdx.y;
  const bool append = k_new != nullptr;
  int64_t t = append ? (int64_t)P.seq_lens[b] : (int64_t)P.seq_lens[b] - 1;
  if (t < 0 || t >= (int64_t)P.max_chunks * kChunk) {  // position outside the block table
    if (tid == 0 && split == 0) set_device_error(kErrChunk);
    t = t < 0 ? 0 : (int64_t)P.max_chunks * kChunk - 1;
  }
  const int64_t own = t / kChunk;
  const int K = P.k - 1;
  float* my_ls = wl_s + warp * kMergeCap;
  int* my_lj = wl_j + warp * kMergeCap;

  if (append && split == 0) {
    const int64_t page = page_of(P, b, own);
    if (page >= 0) {
      const int slot = (int)(t % kChunk);
      for (int x = tid; x < P.Hkv * D; x += kScanThreads) {
        const int g = x / D, e = x % D;
        const int64_t ko = page_offset(P, page, 0, g, slot) + e;
        const int64_t vo = page_offset(P, page, 1, g, slot) + e;
        const int64_t src = ((int64_t)b * P.Hkv + g) * D + e;
        if (P.dtype == HILS_F32) {
          ((float*)P.pages)[ko] = ((const float*)k_new)[src];
          ((float*)P.pages)[vo] = ((const float*)v_new)[src];
        } else {
          ((uint16_t*)P.pages)[ko] = ((const uint16_t*)k_new)[src];
          ((uint16_t*)P.pages)[vo] = ((const uint16_t*)v_new)[src];
        }
      }
    }
  }
  if (split == 0 && tid == 0) ws.tpos[b] = (int32_t)t;

  // a1: q~ for every query head of this sequence
  for (int x = tid; x < P.Hq * D; x += kScanThreads)
    sq[x] = load_elem(P.q, P.dtype, (int64_t)b * P.Hq * D + x);
  __syncthreads();
  for (int x = tid; x < P.Hq * P.r; x += kScanThreads) {
    const int h = x / P.r, a = x % P.r;
    float acc = 0.f;
    for (int e = 0; e < D; ++e) acc = fmaf(sq[h * D + e], P.A[e * P.r + a], acc);
    sT[h * kMaxRank + a] = acc;
  }
  __syncthreads();
  for (int x = tid; x < P.Hq * D; x += kScanThreads) {
    const int h = x / D, e = x % D;
    float acc = sq[x];
    for (int a = 0; a < P.r; ++a) acc = fmaf(sT[h * kMaxRank + a], P.Bm[a * D + e], acc);
    sqt[x] = acc;
  }
  __syncthreads();

  // a2: scores of this split's candidate chunks (j < own), all heads
  const int64_t c0 = (int64_t)split * ws.chunks_per_split;
  const int64_t c1 = min(c0 + ws.chunks_per_split, own);
  const int nloc = c1 > c0 ? (int)(c1 - c0) : 0;
  constexpr int TPR = D / 8;  // threads per landmark row, 8 elements (16 bytes of bf16) each
  const int work = nloc * P.Hkv * TPR;
  for (int xb = 0; xb < work; xb += kScanThreads) {
    const int x = xb + tid;
    const bool ok = x < work;
    const int row = x / TPR, part = x % TPR;
    const int jj = row / P.Hkv, g = row % P.Hkv;
    float v[8];
    if (ok) {
      load8(P.landmarks, P.dtype,
            (((int64_t)b * P.max_chunks + c0 + jj) * P.Hkv + g) * D + part * 8, v);
    } else {
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = 0.f;
    }
    for (int hh = 0; hh < P.group; ++hh) {
      const int h = (ok ? g : 0) * P.group + hh;
      const float* qt = sqt + h * D + part * 8;
      float acc = 0.f;
#pragma unroll
      for (int u = 0; u < 8; ++u) acc = fmaf(qt[u], v[u], acc);
#pragma unroll
      for (int o = TPR / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(kFull, acc, o);
      if (ok && part == 0) sS[jj * P.Hq + h] = acc * P.inv_sqrt_d;
    }
  }
  __syncthreads();

  // a3 (local): best k-1 candidates of this split, per head
  float* cs = ws.cand_s + ((int64_t)b * ws.n_split + split) * P.Hq * K;
  int32_t* cj = ws.cand_j + ((int64_t)b * ws.n_split + split) * P.Hq * K;
  for (int h = warp; h < P.Hq && K > 0; h += kScanWarps) {
    float lmax = -INFINITY;
    for (int x = lane; x < nloc; x += 32) lmax = fmaxf(lmax, sS[x * P.Hq + h]);
    const float tau = warp_kth_largest(lmax, K);
    int cnt = 0;
    for (int xb = 0; xb < nloc; xb += 32) {
      const int x = xb + lane;
      const float v = x < nloc ? sS[x * P.Hq + h] : -INFINITY;
      cnt = warp_append(x < nloc && v >= tau, v, (int)(c0 + x), my_ls, my_lj, cnt, kMergeCap);
    }
    __syncwarp();
    float os;
    int oj;
    warp_select(my_ls, my_lj, min(cnt, kMergeCap), K, os, oj);
    if (lane < K) {
      cs[h * K + lane] = os;
      cj[h * K + lane] = oj;
    }
    __syncwarp();
  }

  // tickets: the last CTA to finish a head merges it
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    unsigned long long mask = 0;
    for (int h = 0; h < P.Hq; ++h) {
      const int old = atomicAdd(&ws.tickets[b * P.Hq + h], 1);
      if (old == ws.n_split - 1) mask |= 1ull << h;
    }
    last_mask = mask;
  }
  __syncthreads();
  const unsigned long long mask = last_mask;
  if (mask == 0) return;
  __threadfence();

  // merge: one warp per head this CTA finished last
  for (int h = warp; h < P.Hq; h += kScanWarps) {
    if (!((mask >> h) & 1ull)) continue;
    float os = -INFINITY;
    int oj = -1;
    if (K > 0) {
      const float* all_s = ws.cand_s + (int64_t)b * ws.n_split * P.Hq * K + (int64_t)h * K;
      const int32_t* all_j = ws.cand_j + (int64_t)b * ws.n_split * P.Hq * K + (int64_t)h * K;
      const int64_t sstride = (int64_t)P.Hq * K;  // between splits
      // lower bound from the splits' best entries (each list is sorted)
      float lmax = -INFINITY;
      for (int sp = lane; sp < ws.n_split; sp += 32) lmax = fmaxf(lmax, __ldcg(all_s + sp * sstride));
      const float tau = warp_kth_largest(lmax, K);
      int cnt = 0;
      for (int spb = 0; spb < ws.n_split; spb += 32) {
        const int sp = spb + lane;
        for (int a = 0; a < K; ++a) {
          float v = -INFINITY;
          int vj = -1;
          if (sp < ws.n_split) {
            v = __ldcg(all_s + sp * sstride + a);
            vj = __ldcg(all_j + sp * sstride + a);
          }
          const bool keep = sp < ws.n_split && vj >= 0 && v >= tau;
          if (!__any_sync(kFull, keep)) break;  // lists are sorted: nothing later survives
          cnt = warp_append(keep, v, vj, my_ls, my_lj, cnt, kMergeCap);
        }
      }
      __syncwarp();
      if (cnt <= kMergeCap) {
        warp_select(my_ls, my_lj, cnt, K, os, oj);
      } else {
        // more survivors than fit (heavily tied scores): select from all lists in two steps
        // of kMergeCap entries each, carrying the best K between steps
        int carried = 0;
        float cs_ = -INFINITY;
        int cj_ = -1;
        const int total = ws.n_split * K;
        for (int x0 = 0; x0 < total; x0 += kMergeCap - 32) {
          __syncwarp();
          int c = 0;
          if (carried) {
            c = warp_append(lane < K && cj_ >= 0, cs_, cj_, my_ls, my_lj, 0, kMergeCap);
          }
          for (int xb = x0; xb < min(x0 + kMergeCap - 32, total); xb += 32) {
            const int x = xb + lane;
            const bool in = x < min(x0 + kMergeCap - 32, total);
            const int sp = x / K, a = x % K;
            float v = -INFINITY;
            int vj = -1;
            if (in) {
              v = __ldcg(all_s + sp * sstride + a);
              vj = __ldcg(all_j + sp * sstride + a);
            }
            c = warp_append(in && vj >= 0, v, vj, my_ls, my_lj, c, kMergeCap);
          }
          __syncwarp();
          warp_select(my_ls, my_lj, min(c, kMergeCap), K, cs_, cj_);
          carried = 1;
        }
        os = cs_;
        oj = cj_;
      }
    }
    // own chunk score
    const int g = h / P.group;
    float acc = 0.f;
    for (int e = lane; e < D; e += 32)
      acc = fmaf(sqt[h * D + e],
                 load_elem(P.landmarks, P.dtype,
                           (((int64_t)b * P.max_chunks + own) * P.Hkv + g) * D + e),
                 acc);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(kFull, acc, o);
    const float s_own = acc * P.inv_sqrt_d;
    // a4: slot 0 = own, slots 1.. = merged list; lane a holds slot a
    const float sh_s = __shfl_sync(kFull, os, (lane + 31) & 31);
    const int sh_j = __shfl_sync(kFull, oj, (lane + 31) & 31);
    const float my_s = lane == 0 ? s_own : sh_s;
    const int my_j = lane == 0 ? (int)own : sh_j;
    const bool live = lane < P.k && my_j >= 0;
    float m = live ? my_s : -INFINITY;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, o));
    const float ex = live ? __expf(my_s - m) : 0.f;
    float z = ex;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(kFull, z, o);
    if (lane < P.k) {
      const int64_t o = ((int64_t)b * P.Hq + h) * P.k + lane;
      const int jv = live ? my_j : -1;
      const float wv = live ? ex / z : 0.f;
      ws.idx[o] = jv;
      ws.w[o] = wv;
      if (idx_out) idx_out[o] = jv;
      if (w_out) w_out[o] = wv;
    }
    if (lane == 0) ws.tickets[b * P.Hq + h] = 0;
    __syncwarp();
  }
  // the CTA that merges the last head advances the sequence length
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const int n_done = __popcll(mask);
    int32_t* done = ws.tickets + 2 * P.B * P.Hq + b;
    const int old = atomicAdd(done, n_done);
    if (old + n_done == P.Hq) {
      if (append) P.seq_lens[b] = (int32_t)(t + 1);
      *done = 0;
    }
  }
}

template <int D>
__global__ void __launch_bounds__(D) attend_kernel(Params P, DecodeWs ws, void* out) {
  __shared__ float sp[kChunk];
  __shared__ float sq[D];
  __shared__ float red[4];
  __shared__ int last;
  const int tid = threadIdx.x;
  const int slot = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int g = h / P.group;
  const int64_t bh = (int64_t)b * P.Hq + h;
  const int32_t j = ws.idx[bh * P.k + slot];
  const float wj = ws.w[bh * P.k + slot];
  const int64_t t = ws.tpos[b];
  float* part = ws.part + (bh * P.k + slot) * D;
  sq[tid] = load_elem(P.q, P.dtype, bh * D + tid);
  __syncthreads();
  if (j >= 0) {
    const int64_t page = page_of(P, b, j);
    const int nk = (j == t / kChunk) ? (int)(t - (int64_t)j * kChunk + 1) : kChunk;
    const bool have = page >= 0 && tid < kChunk && tid < nk;
    float s = -INFINITY;
    if (have) {
      const int64_t ko = page_offset(P, page, 0, g, tid);
      float acc = 0.f;
      for (int e = 0; e < D; e += 8) {
        float kv[8];
        load8(P.pages, P.dtype, ko + e, kv);
#pragma unroll
        for (int u = 0; u < 8; ++u) acc = fmaf(sq[e + u], kv[u], acc);
      }
      s = acc * P.inv_sqrt_d;
    }
    // softmax over the keys held by threads 0..63
    float m = s;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, o));
    if ((tid & 31) == 0 && tid < kChunk) red[tid >> 5] = m;
    __syncthreads();
    m = fmaxf(red[0], red[1]);
    const float ex = have ? __expf(s - m) : 0.f;
    float z = ex;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(kFull, z, o);
    if ((tid & 31) == 0 && tid < kChunk) red[2 + (tid >> 5)] = z;
    if (tid < kChunk) sp[tid] = ex;
    __syncthreads();
    const float l = red[2] + red[3];
    float o = 0.f;
    if (page >= 0) {
      const int64_t vo = page_offset(P, page, 1, g, 0) + tid;
      for (int kk = 0; kk < nk; ++kk)
        o = fmaf(sp[kk], load_elem(P.pages, P.dtype, vo + (int64_t)kk * D), o);
    }
    part[tid] = l > 0.f ? o * (wj / l) : 0.f;
  } else {
    part[tid] = 0.f;
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const int old = atomicAdd(&ws.tickets[P.B * P.Hq + bh], 1);
    last = old == P.k - 1;
  }
  __syncthreads();
  if (!last) return;
  __threadfence();
  float acc = 0.f;
  for (int a = 0; a < P.k; ++a) acc += __ldcg(ws.part + (bh * P.k + a) * D + tid);
  store_elem(out, P.dtype, bh * D + tid, acc);
  if (tid == 0) ws.tickets[P.B * P.Hq + bh] = 0;
}

template <int D>
size_t scan_smem(const Params& P, const DecodeWs& ws) {
  return (size_t)(2 * P.Hq * D + P.Hq * kMaxRank + ws.chunks_per_split * P.Hq) * 4 +
         (size_t)kScanWarps * kMergeCap * 8;
}

template <int D>
cudaError_t run_decode(const Params& P, const void* k_new, const void* v_new, void* out,
                       int32_t* idx_out, float* w_out, const DecodeWs& ws, cudaStream_t s) {
  const size_t smem = scan_smem<D>(P, ws);
  cudaError_t e = cudaFuncSetAttribute(scan_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  {
    HILS_PROFILE("decode.scan", s);
    scan_kernel<D><<<dim3(ws.n_split, P.B), kScanThreads, smem, s>>>(P, k_new, v_new, ws,
                                                                       idx_out, w_out);
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  {
    HILS_PROFILE("decode.attend", s);
    attend_kernel<D><<<dim3(P.k, P.Hq, P.B), D, 0, s>>>(P, ws, out);
  }
  return cudaGetLastError();
}

}  // namespace

static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Split the chunk range so that about two CTAs per SM scan landmarks, with
// between 64 and kMaxSplitChunks chunks (a multiple of 32) per CTA.
static void pick_split(const Params& P, DecodeWs* w) {
  const int64_t target_ctas = 296;
  int64_t per_b = target_ctas / (P.B > 0 ? P.B : 1);
  if (per_b < 1) per_b = 1;
  int64_t cps = (P.max_chunks + per_b - 1) / per_b;
  cps = (cps + 31) / 32 * 32;
  if (cps < 64) cps = 64;
  if (cps > kMaxSplitChunks) cps = kMaxSplitChunks;
  w->chunks_per_split = (int)cps;
  w->n_split = (int)((P.max_chunks + cps - 1) / cps);
  if (w->n_split < 1) w->n_split = 1;
}

size_t decode_ws_bytes(const Params& P, DecodeWs* out, char* base) {
  DecodeWs w{};
  pick_split(P, &w);
  const int K = P.k - 1 > 0 ? P.k - 1 : 1;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    char* p = base ? base + off : nullptr;
    off += align256(bytes);
    return p;
  };
  const int64_t nc = (int64_t)P.B * w.n_split * P.Hq * K;
  w.cand_s = (float*)take(sizeof(float) * nc);
  w.cand_j = (int32_t*)take(sizeof(int32_t) * nc);
  w.idx = (int32_t*)take(sizeof(int32_t) * P.B * P.Hq * P.k);
  w.w = (float*)take(sizeof(float) * P.B * P.Hq * P.k);
  w.part = (float*)take(sizeof(float) * P.B * P.Hq * P.k * P.d);
  w.tickets = (int32_t*)take(sizeof(int32_t) * (2 * P.B * P.Hq + P.B));
  w.tpos = (int32_t*)take(sizeof(int32_t) * P.B);
  if (out) *out = w;
  return off;
}

cudaError_t launch_decode(const Params& P, const void* k_new, const void* v_new, void* out,
                          int32_t* idx_out, float* w_out, const DecodeWs& ws, cudaStream_t s) {
  return P.d == 64 ? run_decode<64>(P, k_new, v_new, out, idx_out, w_out, ws, s)
                   : run_decode<128>(P, k_new, v_new, out, idx_out, w_out, ws, s);
}

}  // namespace hils
