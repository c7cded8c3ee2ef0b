// Decode step (a8): append, calibration, landmark scan, selection, split-k
// chunk attention, as two kernels; the second is launched as a programmatic
// dependent of the first (it may start early and waits for it before reading
// its results).
//
//   scan    grid (n_split, Hkv, B), 256 threads.  A CTA owns one KV head and a
//           contiguous range of chunks of one sequence.  Every thread first
//           issues its 256 bytes of landmark loads and the loads of A, B and
//           the group's queries; q~ = q + (q A) B of the group's query heads is
//           computed while the landmarks land, then every chunk of the range is
//           scored.  Per query head, each warp sorts its part of the range
//           (warp bitonic sort and merges) and warp 0 merges the warps' lists
//           into the range's best k-1, written out best first.  The last CTA of
//           a (sequence, KV head) -- one ticket per CTA -- merges the ranges'
//           lists into the head's best k-1, adds the own chunk (its score from
//           the own landmark), and writes the selection and the fusion weights.
//           The first CTA of a (sequence, KV head) appends k_t and v_t.
//   attend  grid (k, Hq, B), 128 threads.  The CTA of a (sequence, head, slot)
//           attends to the slot's chunk: K and V staged in shared memory,
//           softmax (keys after the query masked in the own chunk), P.V, the
//           weighted partial to the workspace.  The last CTA of a (sequence,
//           head) sums the k partials in slot order (deterministic); the last
//           head of a sequence advances seq_lens.
#include <cfloat>

#include "hils_common.cuh"
#include "tc_common.cuh"

namespace hils {
namespace {

constexpr int kScanThreads = 256;
constexpr int kScanWarps = kScanThreads / 32;
constexpr int kAttThreads = 128;
constexpr unsigned kFull = 0xffffffffu;

// Selection keys.  A score maps to an unsigned key that orders like the score
// (-0 taken as +0); key 0 means "no entry" and lies below every real score, and
// -inf (a chunk that is not a candidate) maps to it as well.  Among equal keys
// the lower chunk index ranks higher.
__device__ __forceinline__ uint32_t score_key(float s) {
  if (s == -INFINITY) return 0u;
  const uint32_t u = __float_as_uint(s + 0.f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_score(uint32_t u) {
  return u == 0u ? -INFINITY : __uint_as_float((u & 0x80000000u) ? (u & 0x7FFFFFFFu) : ~u);
}

// The best (key, chunk) offered by the warp's lanes: the largest key, and among
// lanes holding it the lowest chunk.  Two warp reductions.
__device__ __forceinline__ void warp_best(uint32_t u, int j, uint32_t& bu, int& bj) {
  bu = __reduce_max_sync(kFull, u);
  bj = (int)__reduce_min_sync(kFull, u == bu ? (uint32_t)j : 0xFFFFFFFFu);
}

// Best k (<= 32) of the V entries each lane holds, by rounds of extraction;
// lane a of the result holds the a-th best (key 0: none).  The entries are
// consumed.
template <int V>
__device__ __forceinline__ void warp_topk(uint32_t (&u)[V], int (&j)[V], int k, uint32_t& ou,
                                          int& oj) {
  const int lane = threadIdx.x & 31;
  ou = 0u;
  oj = INT32_MAX;
  for (int it = 0; it < k; ++it) {
    uint32_t cu = 0u;
    int cj = INT32_MAX;
#pragma unroll
    for (int q = 0; q < V; ++q)
      if (u[q] > cu || (u[q] == cu && j[q] < cj)) {
        cu = u[q];
        cj = j[q];
      }
    uint32_t bu;
    int bj;
    warp_best(cu, cj, bu, bj);
    if (bu == 0u) break;
    if (lane == it) {
      ou = bu;
      oj = bj;
    }
#pragma unroll
    for (int q = 0; q < V; ++q)
      if (u[q] == bu && j[q] == bj) u[q] = 0u;
  }
}

// Best k (<= 32) of n lists sorted best first, each of length k, in shared
// memory (list l at lu[l * k], lj[l * k]); lane a of the result holds the a-th
// best.  Lane x follows lists x, x + 32, ...; hp[] holds the lists' read
// positions (shared memory, n entries, reset here).
__device__ __forceinline__ void warp_merge_lists(const uint32_t* lu, const int* lj, int n, int k,
                                                 int* hp, uint32_t& ou, int& oj) {
  const int lane = threadIdx.x & 31;
  for (int l = lane; l < n; l += 32) hp[l] = 0;
  __syncwarp();
  ou = 0u;
  oj = INT32_MAX;
  for (int it = 0; it < k; ++it) {
    uint32_t cu = 0u;
    int cj = INT32_MAX, cl = -1;
    for (int l = lane; l < n; l += 32) {
      const int p = hp[l];
      if (p >= k) continue;
      const uint32_t u = lu[l * k + p];
      const int j = lj[l * k + p];
      if (u > cu || (u == cu && j < cj)) {
        cu = u;
        cj = j;
        cl = l;
      }
    }
    uint32_t bu;
    int bj;
    warp_best(cu, cj, bu, bj);
    if (bu == 0u) break;
    if (lane == it) {
      ou = bu;
      oj = bj;
    }
    if (cl >= 0 && cu == bu && cj == bj) hp[cl] += 1;   // the owner moves past its entry
    __syncwarp();
  }
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

// Decode position of sequence b: seq_lens[b] when appending, else the last
// token; clamped (and flagged) if it falls outside the block table.
__device__ __forceinline__ int64_t decode_pos(const Params& P, int b, bool append, bool report) {
  int64_t t = append ? (int64_t)P.seq_lens[b] : (int64_t)P.seq_lens[b] - 1;
  if (t < 0 || t >= (int64_t)P.max_chunks * kChunk) {
    if (report) set_device_error(kErrChunk);
    t = t < 0 ? 0 : (int64_t)P.max_chunks * kChunk - 1;
  }
  return t;
}

// Landmark work of one scan thread: 256 bytes of one KV head's landmark rows.
template <int D, int EB>
struct ScanGeo {
  static constexpr int SLICE = 256 / EB;                  // landmark elements per thread
  static constexpr int CPT = SLICE >= D ? SLICE / D : 1;  // chunks per thread
  static constexpr int TPC = SLICE >= D ? 1 : D / SLICE;  // threads per chunk
  static constexpr int EPT = SLICE >= D ? D : SLICE;      // elements per (thread, chunk)
  static constexpr int CPS = kScanThreads * CPT / TPC;    // chunks per CTA
  static constexpr int EPU = 16 / EB;                     // elements per 16-byte load
  static constexpr int UPC = EPT / EPU;                   // 16-byte loads per (thread, chunk)
  static constexpr int SEG = CPS / kScanWarps;            // chunks a warp sorts
};

template <int D>
struct ScanSmem {
  // the last part stages the ranges' lists of one query head for the last CTA:
  // keys, chunks and read positions
  static size_t bytes(int r, int group, int cps, int n_split, int k1) {
    return sizeof(float) * (size_t)(2 * D * r + group * D + group * (D + 4) + group * kMaxRank +
                                    cps * group + 2 * kScanWarps * 32 + D +
                                    n_split * (2 * k1 + 1));
  }
};

template <int D, int EB>
__global__ void __launch_bounds__(kScanThreads, 2)
    scan_kernel(Params P, const void* k_new, const void* v_new, DecodeWs ws, int32_t* idx_out,
                float* w_out) {
  using G = ScanGeo<D, EB>;
  // the attention grid may be scheduled now; it waits for this one before its reads
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  constexpr int QS = D + 4;                        // padded q~ row
  const int group = P.group, K = P.k - 1;
  extern __shared__ float sm[];
  float* sA = sm;                                  // [D][r]
  float* sB = sA + D * P.r;                        // [r][D]
  float* sq = sB + P.r * D;                        // [group][D] raw q
  float* sqt = sq + group * D;                     // [group][QS] q~
  float* sT = sqt + group * QS;                    // [group][kMaxRank] q A
  float* sS = sT + group * kMaxRank;               // [CPS][group] scores
  uint32_t* lu = reinterpret_cast<uint32_t*>(sS + G::CPS * group);  // [kScanWarps][k-1] warp lists
  int* lj = reinterpret_cast<int*>(lu + kScanWarps * 32);           // chunks of those
  float* slm = reinterpret_cast<float*>(lj + kScanWarps * 32);      // [D] own chunk's landmark
  uint32_t* mu = reinterpret_cast<uint32_t*>(slm + D);  // [n_split][k-1] ranges' lists (last CTA)
  int* mj = reinterpret_cast<int*>(mu + ws.n_split * K);
  int* mhp = mj + ws.n_split * K;                       // [max(n_split, warps)] read positions
  __shared__ int last;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const bool append = ws.append != 0;
  const int64_t t = decode_pos(P, b, append, tid == 0 && split == 0 && g == 0);
  const int64_t own = t / kChunk;
  const int64_t c0 = (int64_t)split * G::CPS;
  const int cl0 = G::TPC == 1 ? tid * G::CPT : tid / G::TPC;   // first local chunk
  const int part = G::TPC == 1 ? 0 : tid % G::TPC;              // element part of the row

  // ---- every load first ---------------------------------------------------------
  uint4 lm[G::CPT][G::UPC];
#pragma unroll
  for (int ci = 0; ci < G::CPT; ++ci) {
    const int64_t j = c0 + cl0 + ci;
    const bool cand = j < own;
    const uint4* src = reinterpret_cast<const uint4*>(
        reinterpret_cast<const uint8_t*>(P.landmarks) +
        ((((int64_t)b * P.max_chunks + (cand ? j : 0)) * P.Hkv + g) * D + part * G::EPT) * EB);
#pragma unroll
    for (int u = 0; u < G::UPC; ++u) lm[ci][u] = cand ? __ldcs(src + u) : make_uint4(0, 0, 0, 0);
  }
  {
    constexpr int NQ = (64 * D / G::EPU + kScanThreads - 1) / kScanThreads;
    const int na = D * P.r / 4, nq = group * D / G::EPU;
    uint4 rq[NQ], rl = make_uint4(0, 0, 0, 0);
    // A and B straight into shared memory (asynchronous copies, no registers)
    for (int x = tid; x < na; x += kScanThreads) {
      tc::cp_async16(tc::smem_u32(sA + 4 * x), reinterpret_cast<const float4*>(P.A) + x, 16u);
      tc::cp_async16(tc::smem_u32(sB + 4 * x), reinterpret_cast<const float4*>(P.Bm) + x, 16u);
    }
    tc::cp_async_commit();
    const uint4* qsrc = reinterpret_cast<const uint4*>(
        reinterpret_cast<const uint8_t*>(P.q) + ((int64_t)b * P.Hq + (int64_t)g * group) * D * EB);
#pragma unroll
    for (int u = 0; u < NQ; ++u) {
      const int x = u * kScanThreads + tid;
      if (x < nq) rq[u] = __ldg(qsrc + x);
    }
    if (tid < D / G::EPU)
      rl = __ldg(reinterpret_cast<const uint4*>(
          reinterpret_cast<const uint8_t*>(P.landmarks) +
          (((int64_t)b * P.max_chunks + own) * P.Hkv + g) * D * EB) + tid);
    // the append: the first CTA of each (sequence, KV head) writes its head's k_t and v_t
    if (append && split == 0 && tid < 2 * (D / G::EPU)) {
      const int64_t page = page_of(P, b, own);
      if (page >= 0) {
        const int kind = tid / (D / G::EPU), x = tid % (D / G::EPU);
        const uint4* src = reinterpret_cast<const uint4*>(
            reinterpret_cast<const uint8_t*>(kind ? v_new : k_new) + ((int64_t)b * P.Hkv + g) * D * EB) + x;
        uint4* dst = reinterpret_cast<uint4*>(
            reinterpret_cast<uint8_t*>(const_cast<void*>(P.pages)) +
            page_offset(P, page, kind, g, (int)(t % kChunk)) * EB) + x;
        *dst = __ldg(src);
      }
    }
#pragma unroll
    for (int u = 0; u < NQ; ++u) {
      const int x = u * kScanThreads + tid;
      if (x < nq) {
        float v[G::EPU];
        unpack16<EB>(rq[u], v);
#pragma unroll
        for (int e = 0; e < G::EPU; ++e) sq[x * G::EPU + e] = v[e];
      }
    }
    if (tid < D / G::EPU) {
      float v[G::EPU];
      unpack16<EB>(rl, v);
#pragma unroll
      for (int e = 0; e < G::EPU; ++e) slm[tid * G::EPU + e] = v[e];
    }
    tc::cp_async_wait<0>();
  }
  __syncthreads();

  // ---- a1: q~ = q + (q A) B of the group's heads --------------------------------
  if (P.r > 0) {
    // t[h][a]: LP lanes per (h, a) pair, each summing a strided part over e
    const int pairs = group * P.r;
    int LP = 32;
    while (LP > 1 && LP * pairs > kScanThreads) LP >>= 1;
    for (int base = 0; base < pairs * LP; base += kScanThreads) {
      const int x = base + tid;
      const int pr = x / LP, sub = x % LP;
      float acc = 0.f;
      if (pr < pairs) {
        const int h = pr / P.r, a = pr % P.r;
        for (int e = sub; e < D; e += LP) acc = fmaf(sq[h * D + e], sA[e * P.r + a], acc);
      }
      for (int o = LP >> 1; o > 0; o >>= 1) acc += __shfl_xor_sync(kFull, acc, o);
      if (pr < pairs && sub == 0) sT[(pr / P.r) * kMaxRank + pr % P.r] = acc;
    }
    __syncthreads();
  }
  for (int x = tid; x < group * D; x += kScanThreads) {
    const int h = x / D, e = x % D;
    float acc = sq[x];
    for (int a = 0; a < P.r; ++a) acc = fmaf(sT[h * kMaxRank + a], sB[a * D + e], acc);
    sqt[h * QS + e] = acc;
  }
  __syncthreads();

  // ---- a2: scores of the range ----------------------------------------------------
#pragma unroll
  for (int ci = 0; ci < G::CPT; ++ci) {
    const int64_t j = c0 + cl0 + ci;
    for (int hh = 0; hh < group; ++hh) {
      const float* qt = sqt + hh * QS + part * G::EPT;
      float acc = 0.f;
#pragma unroll
      for (int u = 0; u < G::UPC; ++u) {
        float lv[G::EPU];
        unpack16<EB>(lm[ci][u], lv);
#pragma unroll
        for (int e = 0; e < G::EPU; e += 4) {
          const float4 q4 = *reinterpret_cast<const float4*>(qt + u * G::EPU + e);
          acc = fmaf(q4.x, lv[e], acc);
          acc = fmaf(q4.y, lv[e + 1], acc);
          acc = fmaf(q4.z, lv[e + 2], acc);
          acc = fmaf(q4.w, lv[e + 3], acc);
        }
      }
#pragma unroll
      for (int o = 1; o < G::TPC; o <<= 1) acc += __shfl_xor_sync(kFull, acc, o);
      if (part == 0) sS[(cl0 + ci) * group + hh] = j < own ? acc * P.inv_sqrt_d : -INFINITY;
    }
  }
  __syncthreads();

  // ---- a3 (range): best k-1 of the range per query head ---------------------------
  // each warp extracts the best k-1 of its part of the range, warp 0 merges the
  // warps' lists
  for (int hh = 0; hh < group && K > 0; ++hh) {
    const int h = g * group + hh;
    constexpr int V = G::SEG >= 32 ? G::SEG / 32 : 1;
    uint32_t u[V];
    int jj[V];
#pragma unroll
    for (int q = 0; q < V; ++q) {
      const int x = q * 32 + lane;
      const int cl = warp * G::SEG + x;
      u[q] = x < G::SEG ? score_key(sS[cl * group + hh]) : 0u;
      jj[q] = (int)(c0 + cl);
    }
    uint32_t ou;
    int oj;
    warp_topk<V>(u, jj, K, ou, oj);
    if (lane < K) {
      lu[warp * K + lane] = ou;
      lj[warp * K + lane] = oj;
    }
    __syncthreads();
    if (warp == 0) {
      warp_merge_lists(lu, lj, kScanWarps, K, mhp, ou, oj);
      if (lane < K) {
        const int64_t o = (((int64_t)b * P.Hq + h) * ws.n_split + split) * K + lane;
        ws.cand_s[o] = key_score(ou);
        ws.cand_j[o] = ou == 0u ? -1 : oj;
      }
    }
    __syncthreads();
  }

  // ---- a3/a4: the last CTA of the (sequence, KV head) merges the ranges -----------
  __threadfence();
  __syncthreads();
  if (tid == 0) last = atomicAdd(&ws.tickets[b * P.Hkv + g], 1) == ws.n_split - 1;
  __syncthreads();
  if (!last) return;
  __threadfence();
  for (int hh = 0; hh < group; ++hh) {
    const int h = g * group + hh;
    const int64_t bh = (int64_t)b * P.Hq + h;
    // the ranges' lists of this head into shared memory
    for (int x = tid; x < ws.n_split * K; x += kScanThreads) {
      const float v = __ldcg(ws.cand_s + bh * ws.n_split * K + x);
      const int vj = __ldcg(ws.cand_j + bh * ws.n_split * K + x);
      mu[x] = vj < 0 ? 0u : score_key(v);
      mj[x] = vj < 0 ? INT32_MAX : vj;
    }
    __syncthreads();
    if (warp == 0) {
      uint32_t ou = 0u;
      int oj = INT32_MAX;
      if (K > 0) warp_merge_lists(mu, mj, ws.n_split, K, mhp, ou, oj);
      // the own chunk's score
      float so = 0.f;
      for (int e = lane; e < D; e += 32) so = fmaf(sqt[hh * QS + e], slm[e], so);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) so += __shfl_xor_sync(kFull, so, o);
      so *= P.inv_sqrt_d;
      // a4: slot 0 = own chunk, slots 1.. = the merged list; lane a holds slot a
      const uint32_t sh_u = __shfl_sync(kFull, ou, (lane + 31) & 31);
      const int sh_j = __shfl_sync(kFull, oj, (lane + 31) & 31);
      const float my_s = lane == 0 ? so : key_score(sh_u);
      const int my_j = lane == 0 ? (int)own : (sh_u == 0u ? -1 : sh_j);
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
        const int64_t o = bh * P.k + lane;
        ws.idx[o] = jv;
        ws.w[o] = wv;
        if (idx_out) idx_out[o] = jv;
        if (w_out) w_out[o] = wv;
      }
    }
    __syncthreads();
  }
  if (tid == 0) ws.tickets[b * P.Hkv + g] = 0;
}

template <int D, int EB>
__global__ void __launch_bounds__(kAttThreads)
    attend_kernel(Params P, DecodeWs ws, void* out) {
  constexpr int EPU = 16 / EB;                 // elements per 16-byte load
  constexpr int KL = D + (EB == 2 ? 8 : 4);    // padded shared-memory row (elements)
  extern __shared__ __align__(16) uint8_t kv_raw[];   // [2][kChunk][KL] elements
  __shared__ float sq[D];
  __shared__ float sp[kChunk];
  __shared__ float red[8];
  __shared__ float half_o[kAttThreads];
  __shared__ int last;
  const int tid = threadIdx.x, lane = tid & 31, wrp = tid >> 5;
  const int slot = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int g = h / P.group;
  const int64_t bh = (int64_t)b * P.Hq + h;
  // this head's query does not depend on the scan
  for (int e = tid; e < D; e += kAttThreads)
    sq[e] = load_elem(P.q, EB == 2 ? HILS_BF16 : HILS_F32, bh * D + e);
  // wait for the scan (programmatic dependent launch: this grid may start early)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int64_t t = decode_pos(P, b, ws.append != 0, false);
  const int64_t own = t / kChunk;
  const int32_t j = __ldcg(ws.idx + bh * P.k + slot);
  const float wj = __ldcg(ws.w + bh * P.k + slot);
  const int64_t page = j >= 0 ? page_of(P, b, j) : -1;

  // ---- a5: attention to this slot's chunk ----------------------------------
  float* part = ws.part + (bh * P.k + slot) * D;
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
  if (tid == 0) {
    ws.tickets[P.B * P.Hq + bh] = 0;
    // every kernel of the step has read seq_lens: the last head of the sequence advances it
    if (ws.append) {
      int32_t* done = ws.tickets + 2 * P.B * P.Hq + b;
      if (atomicAdd(done, 1) == P.Hq - 1) {
        P.seq_lens[b] = (int32_t)(t + 1);
        *done = 0;
      }
    }
  }
}

size_t scan_smem(const Params& P, int D, int cps, int n_split) {
  const int k1 = P.k - 1, ns = n_split > kScanWarps ? n_split : kScanWarps;
  return D == 64 ? ScanSmem<64>::bytes(P.r, P.group, cps, ns, k1)
                 : ScanSmem<128>::bytes(P.r, P.group, cps, ns, k1);
}

// Launch with programmatic stream serialization: the kernel may start while
// the previous one in the stream is still running.
template <typename... Args, typename... Actual>
cudaError_t launch_pdl(void (*kernel)(Args...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t s, Actual... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

template <int D, int EB>
cudaError_t run_decode(const Params& P, const void* k_new, const void* v_new, void* out,
                       int32_t* idx_out, float* w_out, const DecodeWs& ws, cudaStream_t s) {
  cudaError_t e;
  {
    const size_t smem = scan_smem(P, D, ScanGeo<D, EB>::CPS, ws.n_split);
    if ((e = set_smem(scan_kernel<D, EB>, smem)) != cudaSuccess) return e;
    HILS_PROFILE("decode.scan", s);
    scan_kernel<D, EB><<<dim3(ws.n_split, P.Hkv, P.B), kScanThreads, smem, s>>>(
        P, k_new, v_new, ws, idx_out, w_out);
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  {
    const size_t kv_bytes = (size_t)2 * kChunk * (D + (EB == 2 ? 8 : 4)) * EB;
    if ((e = set_smem(attend_kernel<D, EB>, kv_bytes)) != cudaSuccess) return e;
    HILS_PROFILE("decode.attend", s);
    e = launch_pdl(attend_kernel<D, EB>, dim3(P.k, P.Hq, P.B), dim3(kAttThreads), kv_bytes, s, P,
                   ws, out);
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

int chunks_per_split(const Params& P) {
  if (P.dtype == HILS_BF16) return P.d == 64 ? ScanGeo<64, 2>::CPS : ScanGeo<128, 2>::CPS;
  return P.d == 64 ? ScanGeo<64, 4>::CPS : ScanGeo<128, 4>::CPS;
}

}  // namespace

static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

size_t decode_ws_bytes(const Params& P, DecodeWs* out, char* base) {
  DecodeWs w{};
  w.chunks_per_split = chunks_per_split(P);
  w.n_split = (P.max_chunks + w.chunks_per_split - 1) / w.chunks_per_split;
  if (w.n_split < 1) w.n_split = 1;
  const int K = P.k - 1 > 0 ? P.k - 1 : 1;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    char* p = base ? base + off : nullptr;
    off += align256(bytes);
    return p;
  };
  const int64_t nc = (int64_t)P.B * P.Hq * w.n_split * K;
  w.cand_s = (float*)take(sizeof(float) * nc);
  w.cand_j = (int32_t*)take(sizeof(int32_t) * nc);
  w.idx = (int32_t*)take(sizeof(int32_t) * P.B * P.Hq * P.k);
  w.w = (float*)take(sizeof(float) * P.B * P.Hq * P.k);
  w.part = (float*)take(sizeof(float) * P.B * P.Hq * P.k * P.d);
  w.tickets = (int32_t*)take(sizeof(int32_t) * (2 * P.B * P.Hq + P.B));
  if (out) *out = w;
  return off;
}


cudaError_t launch_decode(const Params& P, const void* k_new, const void* v_new, void* out,
                          int32_t* idx_out, float* w_out, const DecodeWs& ws_in, cudaStream_t s) {
  DecodeWs ws = ws_in;
  ws.append = k_new != nullptr;
  if (P.dtype == HILS_BF16)
    return P.d == 64 ? run_decode<64, 2>(P, k_new, v_new, out, idx_out, w_out, ws, s)
                     : run_decode<128, 2>(P, k_new, v_new, out, idx_out, w_out, ws, s);
  return P.d == 64 ? run_decode<64, 4>(P, k_new, v_new, out, idx_out, w_out, ws, s)
                   : run_decode<128, 4>(P, k_new, v_new, out, idx_out, w_out, ws, s);
}

}  // namespace hils
