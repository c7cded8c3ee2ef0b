// Decode step (a8): append, landmark scan, selection, split-k chunk attention.
//
//   scan    grid (n_split, B), 256 threads.  A CTA owns a contiguous range of
//           chunks of one sequence.  Each thread first issues all its 16-byte
//           landmark loads (a 256-byte slice covering whole heads) together
//           with the calibration matrices; q~ is computed for every query head
//           while they land, then the slice is scored.  Each head's best k-1
//           candidates of the range are found by a warp bitonic sort and
//           written out, best first, with the range's best score; the first
//           CTA also writes every head's own-chunk score.  The last CTA of a
//           sequence (one ticket per CTA) advances seq_lens.  No CTA waits.
//   attend  grid (k, Hq, B), 128 threads, launched as a programmatic
//           dependent of the scan.  Every CTA of a (sequence, head) merges that
//           head's ranges itself (the k CTAs of a head do the same merge in
//           parallel rather than one CTA serially):
//             tau = the (k-1)-th largest of the threads' maxima of the ranges'
//                   best scores -- a lower bound of the (k-1)-th best
//                   candidate, since that many distinct candidates reach it;
//             every range's list (sorted) is read only down to tau;
//             the survivors are reduced to the best k-1 by bitonic merges.
//           The own chunk joins them, the fusion weights follow, and the CTA
//           attends to its slot's chunk (K and V staged in shared memory):
//           softmax, P.V, the weighted partial to the workspace; the last CTA
//           of a (sequence, head) sums the k partials in slot order
//           (deterministic).
#include <cfloat>

#include "hils_common.cuh"

namespace hils {
namespace {

constexpr int kScanThreads = 256;
constexpr int kScanWarps = kScanThreads / 32;
constexpr int kAttThreads = 128;
constexpr int kMergeCap = 512;    // survivors a merging warp can hold
constexpr int kMergeGroup = 8;    // ranges a lane reads per round of loads
constexpr unsigned kFull = 0xffffffffu;

// (sa, ja) ranks above (sb, jb): score descending, then chunk index ascending.
__device__ __forceinline__ bool better(float sa, int ja, float sb, int jb) {
  return sa > sb || (sa == sb && ja < jb);
}

// Sorts one (s, j) per lane across the warp, best first (lane 0 = best).
__device__ __forceinline__ void warp_sort(float& s, int& j) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
    for (int m = k >> 1; m > 0; m >>= 1) {
      const float os = __shfl_xor_sync(kFull, s, m);
      const int oj = __shfl_xor_sync(kFull, j, m);
      const bool lower = (lane & m) == 0;
      const bool desc = (lane & k) == 0;        // this block sorts best first
      const bool keep_better = lower == desc;
      const bool take = keep_better ? better(os, oj, s, j) : better(s, j, os, oj);
      if (take) {
        s = os;
        j = oj;
      }
    }
  }
}

// a (sorted best first across lanes) := best 32 of a and b (b sorted best first).
__device__ __forceinline__ void warp_merge(float& as, int& aj, float bs, int bj) {
  const int lane = threadIdx.x & 31;
  const float rs = __shfl_sync(kFull, bs, 31 - lane);
  const int rj = __shfl_sync(kFull, bj, 31 - lane);
  if (better(rs, rj, as, aj)) {   // the elementwise winners form a bitonic sequence
    as = rs;
    aj = rj;
  }
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) {
    const float os = __shfl_xor_sync(kFull, as, m);
    const int oj = __shfl_xor_sync(kFull, aj, m);
    const bool lower = (lane & m) == 0;
    const bool take = lower ? better(os, oj, as, aj) : better(as, aj, os, oj);
    if (take) {
      as = os;
      aj = oj;
    }
  }
}

// Best 32 of n (s, j) entries in shared memory, sorted best first across lanes.
__device__ void warp_top32(const float* s, const int* j, int n, float& os, int& oj) {
  const int lane = threadIdx.x & 31;
  os = -INFINITY;
  oj = INT32_MAX;
  for (int x0 = 0; x0 < n; x0 += 32) {
    float bs = x0 + lane < n ? s[x0 + lane] : -INFINITY;
    int bj = x0 + lane < n ? j[x0 + lane] : INT32_MAX;
    warp_sort(bs, bj);
    if (x0 == 0) {
      os = bs;
      oj = bj;
    } else {
      warp_merge(os, oj, bs, bj);
    }
  }
}

// Appends (s, j) for lanes with keep to a warp-private list; returns the new count.
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

template <int EB>
__device__ __forceinline__ void unpack16(const uint4& u, float* v) {
  if (EB == 2) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      v[2 * a] = __uint_as_float(w[a] << 16);
      v[2 * a + 1] = __uint_as_float(w[a] & 0xFFFF0000u);
    }
  } else {
    v[0] = __uint_as_float(u.x);
    v[1] = __uint_as_float(u.y);
    v[2] = __uint_as_float(u.z);
    v[3] = __uint_as_float(u.w);
  }
}

// D: head dim; EB: element bytes; SLICE: elements per thread (a multiple or a
// divisor of D, and a divisor of Hkv*D).
template <int D, int EB, int SLICE>
__global__ void __launch_bounds__(kScanThreads, 2)
    scan_kernel(Params P, const void* k_new, const void* v_new, DecodeWs ws) {
  constexpr int U = SLICE * EB / 16;               // 16-byte loads per thread
  constexpr int EPU = 16 / EB;                     // elements per 16-byte load
  constexpr int QS = D + 4;                        // padded q~ row (conflict-free float4 reads)
  extern __shared__ float sm[];
  float* sA = sm;                                  // [D][r] calibration A
  float* sB = sA + D * P.r;                        // [r][D] calibration B
  float* sq = sB + P.r * D;                        // [Hq][D] raw q
  float* sqt = sq + P.Hq * D;                      // [Hq][QS] q~
  float* sT = sqt + P.Hq * QS;                     // [Hq][kMaxRank] q A
  float* sS = sT + P.Hq * kMaxRank;                // [chunks_per_split][Hq] scores
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
  const int row = P.Hkv * D;                       // elements of one chunk's landmarks
  const int64_t c0 = (int64_t)split * ws.chunks_per_split;
  const int64_t c1 = min(c0 + ws.chunks_per_split, own);   // candidates j < own
  const int nloc = c1 > c0 ? (int)(c1 - c0) : 0;

  // ---- every load first: landmark slice, calibration matrices, queries -----
  const int64_t s0 = (int64_t)tid * SLICE;          // element offset inside the range
  const bool have = s0 < (int64_t)nloc * row;
  uint4 lm[U];
  {
    const uint4* src = reinterpret_cast<const uint4*>(
        reinterpret_cast<const uint8_t*>(P.landmarks) +
        (((int64_t)b * P.max_chunks + c0) * row + (have ? s0 : 0)) * EB);
#pragma unroll
    for (int u = 0; u < U; ++u) lm[u] = have ? __ldcs(src + u) : make_uint4(0, 0, 0, 0);
  }
  // the own chunk's landmarks (first CTA of the sequence), one 16-byte unit per thread
  const bool own_unit = split == 0 && tid * EPU < row;
  uint4 own_lm = make_uint4(0, 0, 0, 0);
  if (own_unit)
    own_lm = __ldg(reinterpret_cast<const uint4*>(reinterpret_cast<const uint8_t*>(P.landmarks) +
                                                  (((int64_t)b * P.max_chunks + own) * row +
                                                   tid * EPU) * EB));
  for (int x = tid; x < D * P.r; x += kScanThreads) {
    sA[x] = __ldg(P.A + x);
    sB[x] = __ldg(P.Bm + x);
  }
  for (int x = tid; x < P.Hq * D; x += kScanThreads)
    sq[x] = load_elem(P.q, EB == 2 ? HILS_BF16 : HILS_F32, (int64_t)b * P.Hq * D + x);

  if (append && split == 0) {
    const int64_t page = page_of(P, b, own);
    if (page >= 0) {
      const int slot = (int)(t % kChunk);
      for (int x = tid; x < P.Hkv * D; x += kScanThreads) {
        const int g = x / D, e = x % D;
        const int64_t ko = page_offset(P, page, 0, g, slot) + e;
        const int64_t vo = page_offset(P, page, 1, g, slot) + e;
        const int64_t src = ((int64_t)b * P.Hkv + g) * D + e;
        if (EB == 4) {
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
  __syncthreads();

  // ---- a1: q~ = q + (q A) B for every query head -----------------------------
  for (int x = tid; x < P.Hq * P.r; x += kScanThreads) {
    const int h = x / P.r, a = x % P.r;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};   // four independent chains
#pragma unroll
    for (int e = 0; e < D; e += 4) {
#pragma unroll
      for (int u = 0; u < 4; ++u) acc[u] = fmaf(sq[h * D + e + u], sA[(e + u) * P.r + a], acc[u]);
    }
    sT[h * kMaxRank + a] = (acc[0] + acc[1]) + (acc[2] + acc[3]);
  }
  __syncthreads();
  for (int x = tid; x < P.Hq * D; x += kScanThreads) {
    const int h = x / D, e = x % D;
    float acc = sq[x];
    for (int a = 0; a < P.r; ++a) acc = fmaf(sT[h * kMaxRank + a], sB[a * D + e], acc);
    sqt[h * QS + e] = acc;
  }
  __syncthreads();

  // ---- a2: scores of this thread's slice -------------------------------------
  {
    const int jj = (int)(s0 / row);
    const int off = (int)(s0 % row);
    constexpr int HPS = SLICE >= D ? SLICE / D : 1;   // heads in the slice
    constexpr int TPH = SLICE >= D ? 1 : D / SLICE;   // threads sharing one head
    constexpr int EPH = SLICE >= D ? D : SLICE;       // elements of one head in the slice
#pragma unroll
    for (int hs = 0; hs < HPS; ++hs) {
      const int g = off / D + hs;
      const int e0 = SLICE >= D ? 0 : off % D;
      for (int hh = 0; hh < P.group; ++hh) {
        const int h = (have ? g : 0) * P.group + hh;
        const float* qt = sqt + h * QS + e0;
        float acc = 0.f;
#pragma unroll
        for (int u = 0; u < EPH / EPU; ++u) {
          float lv[EPU];
          unpack16<EB>(lm[hs * (EPH / EPU) + u], lv);
#pragma unroll
          for (int e = 0; e < EPU; e += 4) {
            const float4 q4 = *reinterpret_cast<const float4*>(qt + u * EPU + e);
            acc = fmaf(q4.x, lv[e], acc);
            acc = fmaf(q4.y, lv[e + 1], acc);
            acc = fmaf(q4.z, lv[e + 2], acc);
            acc = fmaf(q4.w, lv[e + 3], acc);
          }
        }
#pragma unroll
        for (int o = 1; o < TPH; o <<= 1) acc += __shfl_xor_sync(kFull, acc, o);
        if (have && (tid % TPH) == 0) sS[jj * P.Hq + h] = acc * P.inv_sqrt_d;
      }
    }
  }
  // own chunk scores: one 16-byte unit per thread, partial dots gathered in shared memory
  if (split == 0) {
    float* part = sS + ws.chunks_per_split * P.Hq;   // [Hq][D / EPU] partial dots
    for (int x = tid; x < row / EPU; x += kScanThreads) {
      const uint4 u = x == tid ? own_lm
                               : __ldg(reinterpret_cast<const uint4*>(
                                     reinterpret_cast<const uint8_t*>(P.landmarks) +
                                     (((int64_t)b * P.max_chunks + own) * row + x * EPU) * EB));
      float lv[EPU];
      unpack16<EB>(u, lv);
      const int g = (x * EPU) / D, e0 = (x * EPU) % D;
      for (int hh = 0; hh < P.group; ++hh) {
        const int h = g * P.group + hh;
        float acc = 0.f;
#pragma unroll
        for (int e = 0; e < EPU; ++e) acc = fmaf(sqt[h * QS + e0 + e], lv[e], acc);
        part[h * (D / EPU) + e0 / EPU] = acc;
      }
    }
    __syncthreads();
    for (int h = warp; h < P.Hq; h += kScanWarps) {
      float acc = 0.f;
      for (int u = lane; u < D / EPU; u += 32) acc += part[h * (D / EPU) + u];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(kFull, acc, o);
      if (lane == 0) ws.s_own[(int64_t)b * P.Hq + h] = acc * P.inv_sqrt_d;
    }
  }
  __syncthreads();

  // ---- a3 (local): best k-1 candidates of the range per head ----------------
  if (K > 0) {
    float* cs = ws.cand_s + ((int64_t)b * ws.n_split + split) * P.Hq * K;
    int32_t* cj = ws.cand_j + ((int64_t)b * ws.n_split + split) * P.Hq * K;
    for (int h = warp; h < P.Hq; h += kScanWarps) {
      float bs = -INFINITY;
      int bj = INT32_MAX;
      for (int x0 = 0; x0 < nloc; x0 += 32) {
        float s = x0 + lane < nloc ? sS[(x0 + lane) * P.Hq + h] : -INFINITY;
        int j = x0 + lane < nloc ? (int)(c0 + x0 + lane) : INT32_MAX;
        warp_sort(s, j);
        if (x0 == 0) {
          bs = s;
          bj = j;
        } else {
          warp_merge(bs, bj, s, j);
        }
      }
      if (lane < K) {
        cs[h * K + lane] = bs;
        cj[h * K + lane] = bj == INT32_MAX ? -1 : bj;
      }
      if (lane == 0) ws.best[((int64_t)b * P.Hq + h) * ws.n_split + split] = bs;
    }
  }

  // ---- the last CTA of the sequence advances seq_lens ---------------------
  if (append) {
    __syncthreads();
    if (tid == 0) {
      int32_t* cnt = ws.tickets + 2 * P.B * P.Hq + b;
      const int old = atomicAdd(cnt, 1);
      if (old == ws.n_split - 1) {
        P.seq_lens[b] = (int32_t)(t + 1);
        *cnt = 0;
      }
    }
  }
}

template <int D, int EB>
__global__ void __launch_bounds__(kAttThreads)
    attend_kernel(Params P, DecodeWs ws, void* out, int32_t* idx_out, float* w_out) {
  constexpr int EPU = 16 / EB;                 // elements per 16-byte load
  constexpr int KL = D + (EB == 2 ? 8 : 4);    // padded shared-memory row (elements)
  constexpr int NW = kAttThreads / 32;
  extern __shared__ __align__(16) uint8_t kv_raw[];   // [2][kChunk][KL] elements
  __shared__ float ms[kMergeCap];
  __shared__ int mj[kMergeCap];
  __shared__ float wmax_s[NW][32];
  __shared__ int mcount;
  __shared__ float tau_sh;
  __shared__ int sel_j[kMaxTopK];
  __shared__ float sel_w[kMaxTopK];
  __shared__ float sq[D];
  __shared__ float sp[kChunk];
  __shared__ float red[8];
  __shared__ float half_o[kAttThreads];
  __shared__ int last;
  // wait for the scan (programmatic dependent launch: this grid may start early)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int tid = threadIdx.x, lane = tid & 31, wrp = tid >> 5;
  const int slot = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int g = h / P.group;
  const int64_t bh = (int64_t)b * P.Hq + h;
  const int K = P.k - 1;
  // independent loads first: position, own score, this head's query
  const int64_t t = __ldcg(ws.tpos + b);
  const float s_own = __ldcg(ws.s_own + bh);
  for (int e = tid; e < D; e += kAttThreads)
    sq[e] = load_elem(P.q, EB == 2 ? HILS_BF16 : HILS_F32, bh * D + e);
  const int64_t own = t / kChunk;

  // ---- a3: merge this head's ranges (every CTA of the head does the same) ----
  if (tid == 0) mcount = 0;
  if (K > 0) {
    const float* bests = ws.best + bh * ws.n_split;
    const float* all_s = ws.cand_s + (int64_t)b * ws.n_split * P.Hq * K + (int64_t)h * K;
    const int32_t* all_j = ws.cand_j + (int64_t)b * ws.n_split * P.Hq * K + (int64_t)h * K;
    const int64_t sstride = (int64_t)P.Hq * K;
    float tmax = -INFINITY;
    for (int sp0 = 0; sp0 < ws.n_split; sp0 += kAttThreads * kMergeGroup) {
      float bv[kMergeGroup];
#pragma unroll
      for (int u = 0; u < kMergeGroup; ++u) {
        const int spl = sp0 + u * kAttThreads + tid;
        bv[u] = spl < ws.n_split ? __ldcg(bests + spl) : -INFINITY;
      }
#pragma unroll
      for (int u = 0; u < kMergeGroup; ++u) tmax = fmaxf(tmax, bv[u]);
    }
    float ts = tmax;
    int tj = tid;
    warp_sort(ts, tj);
    wmax_s[wrp][lane] = ts;
    __syncthreads();
    if (wrp == 0) {
      float as = wmax_s[0][lane];
      int aj = lane;
      for (int w2 = 1; w2 < NW; ++w2) warp_merge(as, aj, wmax_s[w2][lane], 32 * w2 + lane);
      const float tau = __shfl_sync(kFull, as, K - 1);
      if (lane == 0) tau_sh = tau;
    }
    __syncthreads();
    const float tau = tau_sh;
    // survivors: each range's sorted list down to tau
    for (int sp0 = 0; sp0 < ws.n_split; sp0 += kAttThreads * kMergeGroup) {
      float bv[kMergeGroup];
#pragma unroll
      for (int u = 0; u < kMergeGroup; ++u) {
        const int spl = sp0 + u * kAttThreads + tid;
        bv[u] = spl < ws.n_split ? __ldcg(bests + spl) : -INFINITY;
      }
#pragma unroll
      for (int u = 0; u < kMergeGroup; ++u) {
        const int spl = sp0 + u * kAttThreads + tid;
        if (spl >= ws.n_split || !(bv[u] >= tau)) continue;
        for (int a0 = 0; a0 < K; a0 += 4) {
          float v4[4];
          int j4[4];
#pragma unroll
          for (int a = 0; a < 4; ++a) {
            v4[a] = a0 + a < K ? __ldcg(all_s + spl * sstride + a0 + a) : -INFINITY;
            j4[a] = a0 + a < K ? __ldcg(all_j + spl * sstride + a0 + a) : -1;
          }
          bool more = true;
#pragma unroll
          for (int a = 0; a < 4; ++a) {
            if (more && j4[a] >= 0 && v4[a] >= tau) {
              const int at = atomicAdd(&mcount, 1);
              if (at < kMergeCap) {
                ms[at] = v4[a];
                mj[at] = j4[a];
              }
            } else {
              more = false;
            }
          }
          if (!more) break;
        }
      }
    }
  }
  __syncthreads();
  if (wrp == 0) {
    float os = -INFINITY;
    int oj = INT32_MAX;
    if (K > 0) {
      const int cnt = mcount;
      if (cnt <= kMergeCap) {
        warp_top32(ms, mj, cnt, os, oj);
      } else {
        // heavily tied scores: every range's list in full, 32 entries at a time
        const int total = ws.n_split * K;
        const float* all_s = ws.cand_s + (int64_t)b * ws.n_split * P.Hq * K + (int64_t)h * K;
        const int32_t* all_j = ws.cand_j + (int64_t)b * ws.n_split * P.Hq * K + (int64_t)h * K;
        const int64_t sstride = (int64_t)P.Hq * K;
        for (int x0 = 0; x0 < total; x0 += 32) {
          const int x = x0 + lane;
          float v = x < total ? __ldcg(all_s + (x / K) * sstride + x % K) : -INFINITY;
          int vj = x < total ? __ldcg(all_j + (x / K) * sstride + x % K) : -1;
          if (vj < 0) {
            v = -INFINITY;
            vj = INT32_MAX;
          }
          warp_sort(v, vj);
          if (x0 == 0) {
            os = v;
            oj = vj;
          } else {
            warp_merge(os, oj, v, vj);
          }
        }
      }
    }
    // a4: slot 0 = own chunk, slots 1.. = the merged list; lane a holds slot a
    const float sh_s = __shfl_sync(kFull, os, (lane + 31) & 31);
    const int sh_j = __shfl_sync(kFull, oj, (lane + 31) & 31);
    const float my_s = lane == 0 ? s_own : sh_s;
    const int my_j = lane == 0 ? (int)own : (sh_j == INT32_MAX ? -1 : sh_j);
    const bool live = lane < P.k && my_j >= 0;
    float m = live ? my_s : -INFINITY;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, o));
    const float ex = live ? __expf(my_s - m) : 0.f;
    float z = ex;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(kFull, z, o);
    if (lane < P.k) {
      const int jv = live ? my_j : -1;
      const float wv = live ? ex / z : 0.f;
      sel_j[lane] = jv;
      sel_w[lane] = wv;
      if (slot == 0) {
        const int64_t o = bh * P.k + lane;
        ws.idx[o] = jv;
        ws.w[o] = wv;
        if (idx_out) idx_out[o] = jv;
        if (w_out) w_out[o] = wv;
      }
    }
  }
  __syncthreads();

  // ---- a5: attention to this slot's chunk ----------------------------------
  const int32_t j = sel_j[slot];
  const float wj = sel_w[slot];
  float* part = ws.part + (bh * P.k + slot) * D;
  const int64_t page = j >= 0 ? page_of(P, b, j) : -1;
  if (page >= 0) {
    // K and V tiles of the chunk into shared memory: every 16-byte load in flight at once
    const uint8_t* kp = reinterpret_cast<const uint8_t*>(P.pages) + page_offset(P, page, 0, g, 0) * EB;
    const uint8_t* vp = reinterpret_cast<const uint8_t*>(P.pages) + page_offset(P, page, 1, g, 0) * EB;
    constexpr int NU = kChunk * D / EPU;     // 16-byte units per tile
    constexpr int PER = 2 * NU / kAttThreads;
    uint4 u4[PER];
#pragma unroll
    for (int a = 0; a < PER; ++a) {
      const int x = a * kAttThreads + tid;
      const int which = x / NU, y = x % NU;
      u4[a] = __ldg(reinterpret_cast<const uint4*>((which ? vp : kp) + (int64_t)y * 16));
    }
#pragma unroll
    for (int a = 0; a < PER; ++a) {
      const int x = a * kAttThreads + tid;
      const int which = x / NU, y = x % NU;
      const int key = y / (D / EPU), c = y % (D / EPU);
      *reinterpret_cast<uint4*>(kv_raw + ((which * kChunk + key) * KL + c * EPU) * EB) = u4[a];
    }
  }
  __syncthreads();
  if (page >= 0) {
    const int nk = (j == own) ? (int)(t - (int64_t)j * kChunk + 1) : kChunk;
    // scores: two threads per key, each half of the dimensions
    const int key = tid >> 1, hf = tid & 1;
    float acc = 0.f;
    const uint8_t* krow = kv_raw + (key * KL + hf * (D / 2)) * EB;
#pragma unroll 8
    for (int e = 0; e < D / 2; ++e) {
      const float kv = EB == 2 ? __uint_as_float(((uint32_t)reinterpret_cast<const uint16_t*>(krow)[e]) << 16)
                               : reinterpret_cast<const float*>(krow)[e];
      acc = fmaf(sq[hf * (D / 2) + e], kv, acc);
    }
    acc += __shfl_xor_sync(kFull, acc, 1);
    const float s = key < nk ? acc * P.inv_sqrt_d : -INFINITY;
    float m = s;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, o));
    if (lane == 0) red[wrp] = m;
    __syncthreads();
    m = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
    const float ex = key < nk ? __expf(s - m) : 0.f;
    if (hf == 0) sp[key] = ex;
    float z = hf == 0 ? ex : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(kFull, z, o);
    if (lane == 0) red[4 + wrp] = z;
    __syncthreads();
    const float l = red[4] + red[5] + red[6] + red[7];
    // P.V: thread -> one output dimension over one part of the keys
    constexpr int KH = kAttThreads / D;       // key groups (2 for D=64, 1 for D=128)
    const int e = tid % D, kg = tid / D;
    float o = 0.f;
    for (int kk = kg * (kChunk / KH); kk < (kg + 1) * (kChunk / KH); ++kk) {
      const uint8_t* vrow = kv_raw + ((kChunk + kk) * KL + e) * EB;
      const float vv = EB == 2 ? __uint_as_float(((uint32_t)*reinterpret_cast<const uint16_t*>(vrow)) << 16)
                               : *reinterpret_cast<const float*>(vrow);
      o = fmaf(sp[kk], vv, o);
    }
    half_o[tid] = o;
    __syncthreads();
    if (tid < D) {
      float tot = 0.f;
#pragma unroll
      for (int a = 0; a < KH; ++a) tot += half_o[a * D + tid];
      part[tid] = l > 0.f ? tot * (wj / l) : 0.f;
    }
  } else {
    for (int e = tid; e < D; e += kAttThreads) part[e] = 0.f;
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
  for (int e = tid; e < D; e += kAttThreads) {
    float acc = 0.f;
    for (int a = 0; a < P.k; ++a) acc += __ldcg(ws.part + (bh * P.k + a) * D + e);
    store_elem(out, EB == 2 ? HILS_BF16 : HILS_F32, bh * D + e, acc);
  }
  if (tid == 0) ws.tickets[P.B * P.Hq + bh] = 0;
}

size_t scan_smem(const Params& P, const DecodeWs& ws, int D) {
  const int epu = P.dtype == HILS_BF16 ? 8 : 4;
  const size_t own_part = (size_t)P.Hq * (D / epu);
  return (size_t)(2 * D * P.r + P.Hq * D + P.Hq * (D + 4) + P.Hq * kMaxRank +
                  ws.chunks_per_split * P.Hq + own_part) * 4;
}

template <int D, int EB, int SLICE>
cudaError_t run_decode_t(const Params& P, const void* k_new, const void* v_new, void* out,
                         int32_t* idx_out, float* w_out, const DecodeWs& ws, cudaStream_t s) {
  const size_t smem = scan_smem(P, ws, D);
  cudaError_t e = cudaFuncSetAttribute(scan_kernel<D, EB, SLICE>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  {
    HILS_PROFILE("decode.scan", s);
    scan_kernel<D, EB, SLICE><<<dim3(ws.n_split, P.B), kScanThreads, smem, s>>>(P, k_new, v_new, ws);
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  {
    HILS_PROFILE("decode.attend", s);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(P.k, P.Hq, P.B);
    cfg.blockDim = dim3(kAttThreads);
    const size_t kv_bytes = (size_t)2 * kChunk * (D + (EB == 2 ? 8 : 4)) * EB;
    e = cudaFuncSetAttribute(attend_kernel<D, EB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kv_bytes);
    if (e != cudaSuccess) return e;
    cfg.dynamicSmemBytes = kv_bytes;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, attend_kernel<D, EB>, P, ws, out, idx_out, w_out);
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// Elements per thread slice: 256 bytes when a chunk's landmark row splits into
// whole slices of that size, else 128 bytes (float32) / 64 elements.
int slice_elems(const Params& P) {
  const int eb = P.dtype == HILS_BF16 ? 2 : 4;
  return (eb == 2 && (P.Hkv * P.d) % 128 == 0) ? 128 : 64;
}

template <int D, int EB>
cudaError_t run_decode(const Params& P, const void* k_new, const void* v_new, void* out,
                       int32_t* idx_out, float* w_out, const DecodeWs& ws, cudaStream_t s) {
  if (slice_elems(P) == 128)
    return run_decode_t<D, EB, 128>(P, k_new, v_new, out, idx_out, w_out, ws, s);
  return run_decode_t<D, EB, 64>(P, k_new, v_new, out, idx_out, w_out, ws, s);
}

}  // namespace

static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// One CTA scans 256 thread slices, i.e. chunks_per_split chunks.
static void pick_split(const Params& P, DecodeWs* w) {
  const int row = P.Hkv * P.d;
  int cps = row > 0 ? kScanThreads * slice_elems(P) / row : 1;
  if (cps < 1) cps = 1;
  w->chunks_per_split = cps;
  w->n_split = (P.max_chunks + cps - 1) / cps;
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
  w.best = (float*)take(sizeof(float) * (int64_t)P.B * P.Hq * w.n_split);
  w.s_own = (float*)take(sizeof(float) * (int64_t)P.B * P.Hq);
  w.idx = (int32_t*)take(sizeof(int32_t) * P.B * P.Hq * P.k);
  w.w = (float*)take(sizeof(float) * P.B * P.Hq * P.k);
  w.part = (float*)take(sizeof(float) * P.B * P.Hq * P.k * P.d);
  w.tickets = (int32_t*)take(sizeof(int32_t) * (2 * P.B * P.Hq + P.B));
  w.tpos = (int32_t*)take(sizeof(int32_t) * P.B);
  if (out) *out = w;
  return off;
}

size_t decode_scan_smem_bytes(const Params& P) {
  DecodeWs w{};
  pick_split(P, &w);
  return scan_smem(P, w, P.d);
}

cudaError_t launch_decode(const Params& P, const void* k_new, const void* v_new, void* out,
                          int32_t* idx_out, float* w_out, const DecodeWs& ws, cudaStream_t s) {
  if (P.dtype == HILS_BF16)
    return P.d == 64 ? run_decode<64, 2>(P, k_new, v_new, out, idx_out, w_out, ws, s)
                     : run_decode<128, 2>(P, k_new, v_new, out, idx_out, w_out, ws, s);
  return P.d == 64 ? run_decode<64, 4>(P, k_new, v_new, out, idx_out, w_out, ws, s)
                   : run_decode<128, 4>(P, k_new, v_new, out, idx_out, w_out, ws, s);
}

}  // namespace hils
