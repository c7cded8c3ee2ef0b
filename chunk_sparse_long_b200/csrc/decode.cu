// Decode step (a8): append, calibration, landmark scan, selection, split-k
// chunk attention, as two kernels; the second is launched as a programmatic
// dependent of the first (it starts early, does what does not depend on the
// selection, and waits for the first before reading its results).
//
//   scan    grid (n_split, Hkv, B), 256 threads.  A CTA owns one KV head and a
//           contiguous range of chunks of one sequence.  One thread starts TMA
//           copies of the range's landmark rows (64 KB, 128-byte swizzle) into
//           shared memory; meanwhile every thread loads A, B, the group's
//           queries and the own landmark, and q~ = q + (q A) B of the group's
//           query heads is computed.  Every chunk of the range is then scored
//           from shared memory.  Per query head, each warp sorts its part of
//           the range with a bitonic network on 64-bit keys (score, then
//           chunk) and the warps' sorted lists are merged pairwise: the range's
//           best k-1, best first.  The last CTA of a (sequence, KV head) -- one
//           ticket per CTA, taken with acquire-release ordering -- merges the
//           ranges' lists the same way, adds the own chunk (its score from the
//           own landmark), writes the selection, the fusion weights and the
//           selected pages, and starts bringing those pages' K and V into L2.
//           The first CTA of a (sequence, KV head) appends k_t and v_t.
//   attend  grid (n_cta, Hq, B) in clusters of n_cta CTAs, one cluster per
//           (sequence, query head); each CTA takes spc slots (128 threads per
//           slot).  The own chunk (slot 0) does not depend on the selection:
//           its attention runs before the wait, with the new token taken from
//           k_new / v_new.  Every other slot stages its chunk's K and V in
//           shared memory, then softmax (keys after the query masked in the own
//           chunk) and P.V.  The weighted slot outputs are summed inside the CTA;
//           every CTA writes its sum into the first CTA's shared memory
//           (distributed shared memory) and arrives on its barrier, and the
//           first CTA adds them up in slot order (deterministic).  The last
//           head of a sequence advances seq_lens.
#include <cooperative_groups.h>

#include <cfloat>

#include "hils_common.cuh"
#include "tc_common.cuh"

namespace cg = cooperative_groups;

namespace hils {
namespace {

constexpr int kScanThreads = 256;
constexpr int kScanWarps = kScanThreads / 32;
constexpr int kThreads = kScanThreads;
constexpr int kWarps = kScanWarps;
constexpr int kSlotThreads = 128;
constexpr unsigned kFull = 0xffffffffu;
constexpr uint32_t kLmBytes = 65536;   // landmark rows staged per scan CTA

// Selection keys.  The high word is the score mapped to an unsigned order
// (-0 taken as +0), the low word ~j, so a larger key ranks higher in (score
// desc, index asc).  Key 0 means "no entry" and lies below every real score;
// -inf (a chunk that is not a candidate) maps to it.
__device__ __forceinline__ uint64_t sel_key(float s, int64_t j) {
  if (s == -INFINITY) return 0ull;
  uint32_t u = __float_as_uint(s + 0.f);
  u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return ((uint64_t)u << 32) | (uint32_t)(0xFFFFFFFFu - (uint32_t)j);
}
__device__ __forceinline__ float key_score(uint64_t key) {
  if (key == 0ull) return -INFINITY;
  const uint32_t u = (uint32_t)(key >> 32);
  return __uint_as_float((u & 0x80000000u) ? (u & 0x7FFFFFFFu) : ~u);
}
__device__ __forceinline__ int key_chunk(uint64_t key) {
  return key == 0ull ? -1 : (int)(0xFFFFFFFFu - (uint32_t)key);
}

__device__ __forceinline__ uint64_t shfl64(uint64_t v, int src) {
  const uint32_t lo = __shfl_sync(kFull, (uint32_t)v, src);
  const uint32_t hi = __shfl_sync(kFull, (uint32_t)(v >> 32), src);
  return ((uint64_t)hi << 32) | lo;
}
__device__ __forceinline__ uint64_t shfl_xor64(uint64_t v, int m) {
  const uint32_t lo = __shfl_xor_sync(kFull, (uint32_t)v, m);
  const uint32_t hi = __shfl_xor_sync(kFull, (uint32_t)(v >> 32), m);
  return ((uint64_t)hi << 32) | lo;
}

// Bitonic sort of the warp's 32 keys (one per lane), descending across lanes.
__device__ __forceinline__ uint64_t warp_sort32(uint64_t v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      const uint64_t y = shfl_xor64(v, j);
      const bool desc = (lane & k) == 0;
      const bool lower = (lane & j) == 0;
      v = (lower == desc) ? (v > y ? v : y) : (v < y ? v : y);
    }
  }
  return v;
}

// The best 32 of two lists sorted descending across lanes, sorted descending:
// the lane-wise maximum of one list and the reversed other is a bitonic
// sequence holding them, which a half-cleaner cascade sorts.
__device__ __forceinline__ uint64_t warp_merge32(uint64_t a, uint64_t b) {
  const int lane = threadIdx.x & 31;
  const uint64_t br = shfl64(b, 31 - lane);
  uint64_t c = a > br ? a : br;
#pragma unroll
  for (int j = 16; j > 0; j >>= 1) {
    const uint64_t y = shfl_xor64(c, j);
    c = ((lane & j) == 0) ? (c > y ? c : y) : (c < y ? c : y);
  }
  return c;
}

// The best 32 of the warp's 32 V keys (v[q] on every lane), sorted descending.
template <int V>
__device__ __forceinline__ uint64_t warp_top32(uint64_t (&v)[V]) {
#pragma unroll
  for (int q = 0; q < V; ++q) v[q] = warp_sort32(v[q]);
#pragma unroll
  for (int w = 1; w < V; w <<= 1)
#pragma unroll
    for (int q = 0; q + w < V; q += 2 * w) v[q] = warp_merge32(v[q], v[q + w]);
  return v[0];
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
// token; clamped (and flagged) if it falls outside [0, limit).  The limit is
// the block table's capacity, or none (kNoLimit) for the global positions of
// context-parallel decode.
constexpr int64_t kNoLimit = INT64_MAX;
__device__ __forceinline__ int64_t decode_pos(const Params& P, int b, bool append, bool report,
                                              int64_t limit) {
  int64_t t = append ? (int64_t)P.seq_lens[b] : (int64_t)P.seq_lens[b] - 1;
  if (t < 0 || t >= limit) {
    if (report) set_device_error(kErrChunk);
    t = t < 0 ? 0 : limit - 1;
  }
  return t;
}

// Ticket of the calling thread on `p`, with acquire-release ordering at device
// scope: the writes this CTA made before it (published to this thread through
// a CTA barrier) are visible to whoever takes a later ticket, and theirs to
// this CTA.
__device__ __forceinline__ int ticket(int32_t* p) {
  int old;
  asm volatile("atom.add.acq_rel.gpu.s32 %0, [%1], 1;" : "=r"(old) : "l"(p) : "memory");
  return old;
}

// Landmark geometry of one CTA: kLmBytes of landmark rows, CPS chunks of one KV
// head, staged as NCB column blocks of CPS rows x 128 bytes (128-byte swizzle).
template <int D, int EB>
struct Geo {
  static constexpr int ROWB = D * EB;                // bytes of one landmark row
  static constexpr int CPS = kLmBytes / ROWB;        // chunks per CTA: 512, 256 or 128
  static constexpr int NCB = ROWB / 128;             // 128-byte column blocks per row
  static constexpr int BOXR = CPS < 256 ? CPS : 256; // rows per TMA box
  static constexpr int NRB = CPS / BOXR;             // boxes along the chunks
  static constexpr int TPC = CPS >= kThreads ? 1 : kThreads / CPS;   // threads per chunk
  static constexpr int CPT = CPS >= kThreads ? CPS / kThreads : 1;   // chunks per thread
  static constexpr int UNITS = ROWB / 16;            // 16-byte units per row
  static constexpr int UPT = UNITS / TPC;            // units per (thread, chunk)
  static constexpr int EPU = 16 / EB;                // elements per unit
  static constexpr int SEG = CPS / kWarps;           // chunks a warp sorts
  static constexpr int V = SEG >= 32 ? SEG / 32 : 1; // keys per lane in the warp sort
};

// Dynamic shared memory of the scan after the 1024-byte-aligned landmark
// block, in this order: A [D][r], B [r][D] (float), raw q [group][D], q~
// [group][D + 4], q A [group][kMaxRank], scores [CPS][group], own landmark
// [D], the warps' lists [kScanWarps][32] (64-bit), and, for the last CTA, the
// ranges' lists of one head [n_split][k-1] (64-bit).
struct ScanSmem {
  int D, r, group, cps, n_split, k;
  __host__ __device__ size_t floats() const {
    return (size_t)2 * D * r + (size_t)group * D + (size_t)group * (D + 4) +
           (size_t)group * kMaxRank + (size_t)cps * group + D;
  }
  __host__ __device__ size_t lists_off() const {
    return kLmBytes + ((floats() * 4 + 15) & ~(size_t)15);
  }
  __host__ __device__ size_t merge_off() const { return lists_off() + kScanWarps * 32 * 8; }
  __host__ __device__ size_t bytes() const {
    return merge_off() + (size_t)n_split * (k > 1 ? k - 1 : 1) * 8 + 1024;   // + alignment slack
  }
};

template <int D, int EB>
__global__ void __launch_bounds__(kThreads, 2)
    scan_kernel(Params P, const __grid_constant__ CUtensorMap tm_lm, const void* k_new,
                const void* v_new, DecodeWs ws, int32_t* idx_out, float* w_out) {
  using G = Geo<D, EB>;
  // the attention grid may be scheduled now; it waits for this one before its reads
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  constexpr int QS = D + 4;                        // padded q~ row
  const int group = P.group, K = P.k - 1;
  const ScanSmem L{D, P.r, group, G::CPS, ws.n_split, P.k};
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t lm_bar;
  __shared__ int last;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~(uintptr_t)1023);
  uint8_t* lmb = smem;                                   // landmark rows (TMA destination)
  float* sA = reinterpret_cast<float*>(smem + kLmBytes); // [D][r]
  float* sB = sA + D * P.r;                              // [r][D]
  float* sq = sB + P.r * D;                              // [group][D] raw q
  float* sqt = sq + group * D;                           // [group][QS] q~
  float* sT = sqt + group * QS;                          // [group][kMaxRank] q A
  float* sS = sT + group * kMaxRank;                     // [CPS][group] scores
  float* slm = sS + G::CPS * group;                      // [D] own chunk's landmark
  uint64_t* wl = reinterpret_cast<uint64_t*>(smem + L.lists_off());   // [kWarps][32]
  uint64_t* ml = reinterpret_cast<uint64_t*>(smem + L.merge_off());   // [n_split][K]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const bool append = ws.append != 0;
  // context-parallel mode: ws.cp_own set (read from the parameter where used)
  const bool report = tid == 0 && split == 0 && g == 0;
  const int64_t t =
      decode_pos(P, b, append, report, ws.cp_own ? kNoLimit : (int64_t)P.max_chunks * kChunk);
  // the own chunk, local to this cache; in context-parallel mode it may lie
  // outside (below 0, or past the cache, where max_chunks stands for it), and
  // the candidates are the local chunks before it in either case
  int64_t own = t / kChunk - ws.chunk_base;
  if (own > P.max_chunks) own = P.max_chunks;
  const int cps = ws.chunks_per_split;            // chunks of this range (<= CPS)
  const int64_t c0 = (int64_t)split * cps;
  const bool any_cand = c0 < own;                 // the range holds a chunk before the own one

  // ---- loads: the landmark rows by TMA, the small inputs by every thread ------
  if (tid == 0) {
    tc::mbar_init(&lm_bar, 1);
    tc::fence_mbar_init();
  }
  __syncthreads();
  if (tid == 0 && any_cand) {
    tc::mbar_arrive_expect_tx(&lm_bar, kLmBytes);
#pragma unroll
    for (int rb = 0; rb < G::NRB; ++rb)
#pragma unroll
      for (int cb = 0; cb < G::NCB; ++cb)
        tc::tma_load_4d(tc::smem_u32(lmb + cb * (G::CPS * 128) + rb * (G::BOXR * 128)), &tm_lm,
                        cb * (128 / EB), g, (int)(c0 + rb * G::BOXR), b, &lm_bar);
  }
  {
    constexpr int NQ = (64 * D / G::EPU + kThreads - 1) / kThreads;
    const int na = D * P.r / 4, nq = group * D / G::EPU;
    // A and B straight into shared memory (asynchronous copies, no registers)
    for (int x = tid; x < na; x += kThreads) {
      tc::cp_async16(tc::smem_u32(sA + 4 * x), reinterpret_cast<const float4*>(P.A) + x, 16u);
      tc::cp_async16(tc::smem_u32(sB + 4 * x), reinterpret_cast<const float4*>(P.Bm) + x, 16u);
    }
    tc::cp_async_commit();
    uint4 rq[NQ], rl = make_uint4(0, 0, 0, 0);
    const uint4* qsrc = reinterpret_cast<const uint4*>(
        reinterpret_cast<const uint8_t*>(P.q) + ((int64_t)b * P.Hq + (int64_t)g * group) * D * EB);
#pragma unroll
    for (int u = 0; u < NQ; ++u) {
      const int x = u * kThreads + tid;
      if (x < nq) rq[u] = __ldg(qsrc + x);
    }
    if (own >= 0 && own < P.max_chunks && tid < D / G::EPU)
      rl = __ldg(reinterpret_cast<const uint4*>(
          reinterpret_cast<const uint8_t*>(P.landmarks) +
          (((int64_t)b * P.max_chunks + own) * P.Hkv + g) * D * EB) + tid);
    // the append: the first CTA of each (sequence, KV head) writes its head's k_t and v_t
    if (append && own >= 0 && own < P.max_chunks && split == 0 && tid < 2 * (D / G::EPU)) {
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
      const int x = u * kThreads + tid;
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
    while (LP > 1 && LP * pairs > kThreads) LP >>= 1;
    for (int base = 0; base < pairs * LP; base += kThreads) {
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
  for (int x = tid; x < group * D; x += kThreads) {
    const int h = x / D, e = x % D;
    float acc = sq[x];
    for (int a = 0; a < P.r; ++a) acc = fmaf(sT[h * kMaxRank + a], sB[a * D + e], acc);
    sqt[h * QS + e] = acc;
  }
  __syncthreads();

  // ---- a2: scores of the range, from the staged landmark rows ---------------------
  bool lm_ok = true;
  if (any_cand) {
    lm_ok = tc::mbar_wait(&lm_bar, 0, wait_limit());
    // a CTA that gave up still lets its copies land before it goes on
    if (!lm_ok) tc::mbar_wait(&lm_bar, 0, kDrainLimitNs);
  }
  if (!lm_ok && tid == 0) set_device_error(kErrTimeout);
#pragma unroll
  for (int ci = 0; ci < G::CPT; ++ci) {
    const int cl = G::TPC == 1 ? tid + ci * kThreads : tid / G::TPC;   // local chunk
    const int part = G::TPC == 1 ? 0 : tid % G::TPC;
    const int64_t j = c0 + cl;
    const bool cand = lm_ok && cl < cps && j < own;
    for (int hh = 0; hh < group; ++hh) {
      float acc = 0.f;
      if (cand) {
        const float* qt = sqt + hh * QS;
#pragma unroll
        for (int v = 0; v < G::UPT; ++v) {
          const int u = part * G::UPT + v;
          const uint4 w4 = *reinterpret_cast<const uint4*>(lmb + (u >> 3) * (G::CPS * 128) +
                                                           tc::swz(cl, u & 7));
          float lv[G::EPU];
          unpack16<EB>(w4, lv);
#pragma unroll
          for (int e = 0; e < G::EPU; e += 4) {
            const float4 q4 = *reinterpret_cast<const float4*>(qt + u * G::EPU + e);
            acc = fmaf(q4.x, lv[e], acc);
            acc = fmaf(q4.y, lv[e + 1], acc);
            acc = fmaf(q4.z, lv[e + 2], acc);
            acc = fmaf(q4.w, lv[e + 3], acc);
          }
        }
      }
#pragma unroll
      for (int o = 1; o < G::TPC; o <<= 1) acc += __shfl_xor_sync(kFull, acc, o);
      if (part == 0) sS[cl * group + hh] = cand ? acc * P.inv_sqrt_d : -INFINITY;
    }
  }
  __syncthreads();

  // ---- a3 (range): best k-1 of the range per query head ---------------------------
  // each warp sorts its part of the range; the warps' lists are merged pairwise
  for (int hh = 0; hh < group && K > 0; ++hh) {
    const int h = g * group + hh;
    uint64_t v[G::V];
#pragma unroll
    for (int q = 0; q < G::V; ++q) {
      const int x = q * 32 + lane;
      const int cl = warp * G::SEG + x;
      v[q] = x < G::SEG ? sel_key(sS[cl * group + hh], ws.chunk_base + c0 + cl) : 0ull;
    }
    wl[warp * 32 + lane] = warp_top32<G::V>(v);
#pragma unroll
    for (int step = 1; step < kWarps; step <<= 1) {
      __syncthreads();
      if ((warp & (2 * step - 1)) == 0)
        wl[warp * 32 + lane] = warp_merge32(wl[warp * 32 + lane], wl[(warp + step) * 32 + lane]);
    }
    __syncthreads();
    if (warp == 0 && lane < K)
      ws.cand[(((int64_t)b * P.Hq + h) * ws.n_split + split) * K + lane] = wl[lane];
    __syncthreads();
  }

  // ---- the last CTA of the (sequence, KV head) takes over -------------------------
  if (tid == 0) last = ticket(&ws.tickets[b * P.Hkv + g]) == ws.n_split - 1;
  __syncthreads();
  if (!last) return;

  for (int hh = 0; hh < group; ++hh) {
    const int h = g * group + hh;
    const int64_t bh = (int64_t)b * P.Hq + h;
    if (K > 0) {
      // the ranges' lists of this head into shared memory, then a tree of merges
      for (int x = tid; x < ws.n_split * K; x += kScanThreads)
        ml[x] = __ldcg(ws.cand + bh * ws.n_split * K + x);
      for (int step = 1; step < ws.n_split; step <<= 1) {
        __syncthreads();
        for (int a = warp * 2 * step; a + step < ws.n_split; a += kScanWarps * 2 * step) {
          const uint64_t x = lane < K ? ml[a * K + lane] : 0ull;
          const uint64_t y = lane < K ? ml[(a + step) * K + lane] : 0ull;
          const uint64_t c = warp_merge32(x, y);
          if (lane < K) ml[a * K + lane] = c;
        }
      }
      __syncthreads();
    }
    if (warp == 0) {
      const uint64_t key = (K > 0 && lane < K) ? ml[lane] : 0ull;
      // the own chunk's score
      float so = 0.f;
      for (int e = lane; e < D; e += 32) so = fmaf(sqt[hh * QS + e], slm[e], so);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) so += __shfl_xor_sync(kFull, so, o);
      so *= P.inv_sqrt_d;
      if (ws.cp_own) {
        // the merged list and the own score leave for the gather across GPUs
        if (K > 0 && lane < K) ws.cp_keys[bh * K + lane] = key;
        if (lane == 0) ws.cp_own[bh] = (own >= 0 && own < P.max_chunks) ? so : -INFINITY;
      } else {
        // a4: slot 0 = own chunk, slots 1.. = the merged list; lane a holds slot a
        const uint64_t sh = shfl64(key, (lane + 31) & 31);
        const float my_s = lane == 0 ? so : key_score(sh);
        const int my_j = lane == 0 ? (int)own : key_chunk(sh);
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
          const int64_t page = live ? page_of(P, b, jv) : -1;
          const int64_t o = bh * P.k + lane;
          ws.idx[o] = jv;
          ws.w[o] = wv;
          ws.page[o] = (int32_t)page;
          if (idx_out) idx_out[o] = jv;
          if (w_out) w_out[o] = wv;
          // the attention kernel reads these pages next: start bringing them into L2
          if (page >= 0 && lane > 0) {
            const uint8_t* base = reinterpret_cast<const uint8_t*>(P.pages);
            tc::bulk_prefetch_l2(base + page_offset(P, page, 0, g, 0) * EB, kChunk * D * EB);
            tc::bulk_prefetch_l2(base + page_offset(P, page, 1, g, 0) * EB, kChunk * D * EB);
          }
        }
      }
    }
    __syncthreads();
  }
  if (tid == 0) ws.tickets[b * P.Hkv + g] = 0;
}

// Shared memory of one slot's K and V tiles: [2][kChunk][KL] elements with a
// padded row of KL elements.
template <int D, int EB>
struct SlotTiles {
  static constexpr int KL = D + (EB == 2 ? 8 : 4);
  static constexpr size_t kBytes = (size_t)2 * kChunk * KL * EB;
};

// Attention of query `sq` to one chunk staged at `kv` (K rows then V rows),
// keys 0 .. nk-1, by the 128 threads of a slot group (index st).  Leaves the
// unnormalised output, dimension st % D, summed over the group's key halves in
// `acc` (valid for st < D) and returns l, the sum of the probabilities.
template <int D, int EB>
__device__ __forceinline__ float chunk_attend(const float* sq, const uint8_t* kv, int nk,
                                              float inv_sqrt_d, float* sp, float* red,
                                              float* half_o, int st, float& acc, int bar_id) {
  using T = SlotTiles<D, EB>;
  const int lane = st & 31, wrp = st >> 5;
  // scores: two threads per key, each half of the dimensions
  const int key = st >> 1, hf = st & 1;
  float a = 0.f;
  const uint8_t* krow = kv + (key * T::KL + hf * (D / 2)) * EB;
#pragma unroll 8
  for (int e = 0; e < D / 2; ++e) {
    const float kv_e = EB == 2 ? __uint_as_float(((uint32_t)reinterpret_cast<const uint16_t*>(krow)[e]) << 16)
                               : reinterpret_cast<const float*>(krow)[e];
    a = fmaf(sq[hf * (D / 2) + e], kv_e, a);
  }
  a += __shfl_xor_sync(kFull, a, 1);
  const float s = key < nk ? a * inv_sqrt_d : -INFINITY;
  float m = s;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, o));
  if (lane == 0) red[wrp] = m;
  tc::named_barrier(bar_id, kSlotThreads);
  m = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  const float ex = key < nk ? __expf(s - m) : 0.f;
  if (hf == 0) sp[key] = ex;
  float z = hf == 0 ? ex : 0.f;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(kFull, z, o);
  if (lane == 0) red[4 + wrp] = z;
  tc::named_barrier(bar_id, kSlotThreads);
  const float l = red[4] + red[5] + red[6] + red[7];
  // P.V: thread -> one output dimension over one part of the keys
  constexpr int KH = kSlotThreads / D;       // key groups (2 for D=64, 1 for D=128)
  const int e = st % D, kg = st / D;
  float o = 0.f;
  for (int kk = kg * (kChunk / KH); kk < (kg + 1) * (kChunk / KH); ++kk) {
    const uint8_t* vrow = kv + ((kChunk + kk) * T::KL + e) * EB;
    const float vv = EB == 2 ? __uint_as_float(((uint32_t)*reinterpret_cast<const uint16_t*>(vrow)) << 16)
                             : *reinterpret_cast<const float*>(vrow);
    o = fmaf(sp[kk], vv, o);
  }
  half_o[st] = o;
  tc::named_barrier(bar_id, kSlotThreads);
  acc = 0.f;
  if (st < D) {
#pragma unroll
    for (int x = 0; x < KH; ++x) acc += half_o[x * D + st];
  }
  return l;
}

// Stages rows [0, 64) of K and V of (page, KV head g) into `kv` with every
// 16-byte load of the slot group in flight at once.
template <int D, int EB>
__device__ __forceinline__ void stage_tiles(const Params& P, int64_t page, int g, uint8_t* kv,
                                            int st) {
  using T = SlotTiles<D, EB>;
  constexpr int EPU = 16 / EB;
  constexpr int NU = kChunk * D / EPU;     // 16-byte units per tile
  constexpr int PER = 2 * NU / kSlotThreads;
  const uint8_t* kp = reinterpret_cast<const uint8_t*>(P.pages) + page_offset(P, page, 0, g, 0) * EB;
  const uint8_t* vp = reinterpret_cast<const uint8_t*>(P.pages) + page_offset(P, page, 1, g, 0) * EB;
  uint4 u4[PER];
#pragma unroll
  for (int a = 0; a < PER; ++a) {
    const int x = a * kSlotThreads + st;
    const int which = x / NU, y = x % NU;
    u4[a] = __ldcg(reinterpret_cast<const uint4*>((which ? vp : kp) + (int64_t)y * 16));
  }
#pragma unroll
  for (int a = 0; a < PER; ++a) {
    const int x = a * kSlotThreads + st;
    const int which = x / NU, y = x % NU;
    const int key = y / (D / EPU), c = y % (D / EPU);
    *reinterpret_cast<uint4*>(kv + ((which * kChunk + key) * T::KL + c * EPU) * EB) = u4[a];
  }
}

template <int D, int EB>
__global__ void __launch_bounds__(kSlotThreads * 2)
    attend_kernel(Params P, DecodeWs ws, const void* k_new, const void* v_new, void* out,
                  int spc) {
  using T = SlotTiles<D, EB>;
  constexpr int EPU = 16 / EB;
  extern __shared__ __align__(16) uint8_t kv_raw[];   // spc x [2][kChunk][KL] elements
  __shared__ float sq[D];
  __shared__ float sp[2][kChunk];
  __shared__ float red[2][8];
  __shared__ float half_o[2][kSlotThreads];
  __shared__ float part[2][D];
  __shared__ float cpart[16][D];   // rank 0: every CTA's sum, at its rank
  __shared__ uint64_t cpart_bar;   // rank 0: one arrival per other CTA of the cluster
  cg::cluster_group cluster = cg::this_cluster();
  const int tid = threadIdx.x;
  const int sg = tid / kSlotThreads, st = tid % kSlotThreads;
  const int rank = (int)cluster.block_rank();
  const int n_cta = (int)cluster.num_blocks();
  const int h = blockIdx.y, b = blockIdx.z;
  const int g = h / P.group;
  const int64_t bh = (int64_t)b * P.Hq + h;
  const int slot = rank * spc + sg;
  const bool active = slot < P.k;
  const bool append = ws.append != 0;
  uint8_t* kv = kv_raw + sg * T::kBytes;
  const int bar_id = 1 + sg;
  // none of this depends on the scan: the query, the position, and the own chunk
  for (int e = tid; e < D; e += blockDim.x)
    sq[e] = load_elem(P.q, EB == 2 ? HILS_BF16 : HILS_F32, bh * D + e);
  const bool cp = ws.cp_partial != nullptr;       // context-parallel mode
  const int64_t t =
      decode_pos(P, b, append, false, cp ? kNoLimit : (int64_t)P.max_chunks * kChunk);
  const int64_t own = t / kChunk;                  // global chunk index
  const int64_t own_l = own - ws.chunk_base;       // in this cache
  const int tr = (int)(t % kChunk);
  if (rank == 0 && tid == 0) {
    tc::mbar_init(&cpart_bar, n_cta > 1 ? n_cta - 1 : 1);
    tc::fence_mbar_init();
  }
  // the barrier exists before any CTA of the cluster can arrive on it
  cluster.sync();
  float acc = 0.f, l = 0.f;
  bool have = false;
  if (active && slot == 0 && own_l >= 0 && own_l < P.max_chunks) {
    const int64_t page = page_of(P, b, own_l);
    if (page >= 0) {
      stage_tiles<D, EB>(P, page, g, kv, st);
      tc::named_barrier(bar_id, kSlotThreads);
      // the new token is written by the scan: take it from the inputs
      if (append && st < 2 * (D / EPU)) {
        const int kind = st / (D / EPU), x = st % (D / EPU);
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(
            reinterpret_cast<const uint8_t*>(kind ? v_new : k_new) + ((int64_t)b * P.Hkv + g) * D * EB) + x);
        *reinterpret_cast<uint4*>(kv + ((kind * kChunk + tr) * T::KL + x * EPU) * EB) = v;
      }
      tc::named_barrier(bar_id, kSlotThreads);
      l = chunk_attend<D, EB>(sq, kv, tr + 1, P.inv_sqrt_d, sp[sg], red[sg], half_o[sg], st, acc,
                              bar_id);
      have = true;
    }
  }
  // wait for the scan (programmatic dependent launch: this grid started early)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  float wj = 0.f;
  if (active) {
    wj = __ldcg(ws.w + bh * P.k + slot);
    if (slot > 0) {
      const int32_t j = __ldcg(ws.idx + bh * P.k + slot);
      int64_t page = -1;
      if (!cp)
        page = __ldcg(ws.page + bh * P.k + slot);
      else if (j >= 0 && j - ws.chunk_base >= 0 && j - ws.chunk_base < P.max_chunks)
        page = page_of(P, b, j - ws.chunk_base);   // a selected chunk held here
      if (page >= 0) {
        stage_tiles<D, EB>(P, page, g, kv, st);
        tc::named_barrier(bar_id, kSlotThreads);
        l = chunk_attend<D, EB>(sq, kv, j == own ? tr + 1 : kChunk, P.inv_sqrt_d, sp[sg],
                                red[sg], half_o[sg], st, acc, bar_id);
        have = true;
      }
    }
  }
  if (st < D) part[sg][st] = (have && l > 0.f) ? acc * (wj / l) : 0.f;
  __syncthreads();
  // this CTA's slots summed in slot order, into rank 0's shared memory
  float* dst = cluster.map_shared_rank(&cpart[0][0], 0) + rank * D;
  if (tid < D) {
    float c = 0.f;
    for (int x = 0; x < spc; ++x) c += part[x][tid];
    dst[tid] = c;
  }
  if (rank != 0) {
    __syncthreads();
    if (tid == 0) tc::mbar_arrive_remote_cluster(&cpart_bar, 0);
    return;
  }
  // rank 0: the cluster's sums in rank (= slot) order, once every other CTA's has landed
  bool ok = true;
  if (n_cta > 1) ok = tc::mbar_wait_cluster(&cpart_bar, 0);
  if (!ok) {
    if (tid == 0) set_device_error(kErrTimeout);
    return;
  }
  __syncthreads();
  if (tid < D) {
    float o = 0.f;
    for (int r = 0; r < n_cta; ++r) o += cpart[r][tid];
    if (cp)
      ws.cp_partial[bh * D + tid] = o;
    else
      store_elem(out, EB == 2 ? HILS_BF16 : HILS_F32, bh * D + tid, o);
  }
  // every kernel of the step has read seq_lens: the last head of the sequence advances it
  if (tid == 0 && append && !cp) {
    __threadfence();
    int32_t* done = ws.tickets + P.B * P.Hkv + b;
    if (atomicAdd(done, 1) == P.Hq - 1) {
      P.seq_lens[b] = (int32_t)(t + 1);
      *done = 0;
    }
  }
}

// Launch with programmatic stream serialization (the kernel may start while
// the previous one in the stream is still running) and, when cluster > 1, in
// clusters of `cluster` CTAs along x.
template <typename... Args, typename... Actual>
cudaError_t launch_pdl(void (*kernel)(Args...), dim3 grid, dim3 block, size_t smem, int cluster,
                       cudaStream_t s, Actual... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = cluster;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Slots per attention CTA and CTAs per cluster: at most two slots per CTA, at
// most 8 CTAs per cluster up to k = 16 (16, a non-portable size, above).
void attend_shape(int k, int* spc, int* n_cta) {
  *n_cta = k <= 8 ? k : (k <= 16 ? 8 : 16);
  *spc = (k + *n_cta - 1) / *n_cta;
}

// The scan (a1-a4): one CTA per (chunk range, KV head, sequence).
template <int D, int EB>
cudaError_t launch_scan(const Params& P, const void* k_new, const void* v_new, const DecodeWs& ws,
                        int32_t* idx_out, float* w_out, cudaStream_t s) {
  using G = Geo<D, EB>;
  cudaError_t e;
  CUtensorMap tm;
  const uint64_t dims[4] = {(uint64_t)D, (uint64_t)P.Hkv, (uint64_t)P.max_chunks, (uint64_t)P.B};
  const uint64_t strides[3] = {(uint64_t)D * EB, (uint64_t)P.Hkv * D * EB,
                               (uint64_t)P.max_chunks * P.Hkv * D * EB};
  const uint32_t box[4] = {128u / EB, 1, (uint32_t)G::BOXR, 1};
  if ((e = encode_tmap(&tm, EB == 2 ? HILS_BF16 : HILS_F32, 4, P.landmarks, dims, strides, box)) !=
      cudaSuccess)
    return e;
  const size_t smem = ScanSmem{D, P.r, P.group, G::CPS, ws.n_split, P.k}.bytes();
  if ((e = set_smem(scan_kernel<D, EB>, smem)) != cudaSuccess) return e;
  HILS_PROFILE(ws.cp_own ? "decode_cp.candidates" : "decode.scan", s);
  scan_kernel<D, EB><<<dim3(ws.n_split, P.Hkv, P.B), kScanThreads, smem, s>>>(P, tm, k_new, v_new,
                                                                             ws, idx_out, w_out);
  return cudaGetLastError();
}

// The attention (a5, a6): one cluster of CTAs per (query head, sequence),
// launched early (programmatic dependent launch) behind the previous kernel.
template <int D, int EB>
cudaError_t launch_attend(const Params& P, const DecodeWs& ws, const void* k_new,
                          const void* v_new, void* out, cudaStream_t s) {
  int spc, n_cta;
  attend_shape(P.k, &spc, &n_cta);
  const size_t kv_bytes = (size_t)spc * SlotTiles<D, EB>::kBytes;
  cudaError_t e;
  if ((e = set_smem(attend_kernel<D, EB>, kv_bytes)) != cudaSuccess) return e;
  if (n_cta > 8) {
    static bool np_set[2][2] = {};   // one flag per instantiation
    bool& done = np_set[D == 128][EB == 4];
    if (!done) {
      e = cudaFuncSetAttribute(attend_kernel<D, EB>,
                               cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      if (e != cudaSuccess) return e;
      done = true;
    }
  }
  HILS_PROFILE(ws.cp_partial ? "decode_cp.attend" : "decode.attend", s);
  e = launch_pdl(attend_kernel<D, EB>, dim3(n_cta, P.Hq, P.B), dim3(kSlotThreads * spc), kv_bytes,
                 n_cta, s, P, ws, k_new, v_new, out, spc);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int D, int EB>
cudaError_t run_decode(const Params& P, const void* k_new, const void* v_new, void* out,
                       int32_t* idx_out, float* w_out, const DecodeWs& ws, cudaStream_t s) {
  cudaError_t e = launch_scan<D, EB>(P, k_new, v_new, ws, idx_out, w_out, s);
  if (e != cudaSuccess) return e;
  return launch_attend<D, EB>(P, ws, k_new, v_new, out, s);
}

// ---- context-parallel decode ---------------------------------------------
// One sequence's chunks spread over several GPUs: this GPU holds the chunks
// chunk_base .. chunk_base + P.max_chunks - 1 (its block table, pages and
// landmarks are indexed by local chunk); seq_lens holds the global positions.
// The selection exchanges only each GPU's best k-1 keys and the own chunk's
// score; the output, only each GPU's weighted sum over the selected chunks it
// holds.  The scan and the attention are the kernels above in their
// context-parallel mode; the selection from the gathered lists and the final
// cast are below.

// Per (query head, sequence), one warp: the global selection from the
// gathered lists [world][B][Hq][k-1] and own scores [world][B][Hq] -- the
// same slot order and weights as hils_decode.
__global__ void __launch_bounds__(32) cp_select_kernel(Params P, int world, const uint64_t* keys,
                                                       const float* own_scores, bool append,
                                                       int32_t* idx, float* w) {
  const int h = blockIdx.x, b = blockIdx.y, lane = threadIdx.x;
  const int K = P.k - 1;
  const int64_t bh = (int64_t)b * P.Hq + h, nbh = (int64_t)P.B * P.Hq;
  const int64_t own = decode_pos(P, b, append, lane == 0, kNoLimit) / kChunk;
  uint64_t c = 0ull;
  float so = -INFINITY;
  for (int r = 0; r < world; ++r) {
    const uint64_t x = (K > 0 && lane < K) ? keys[(r * nbh + bh) * K + lane] : 0ull;
    c = r == 0 ? x : warp_merge32(c, x);
    so = fmaxf(so, own_scores[r * nbh + bh]);
  }
  if (so == -INFINITY && lane == 0) set_device_error(kErrChunk);   // no GPU holds the own chunk
  // slot 0 = own chunk, slots 1.. = the merged list; lane a holds slot a
  const uint64_t sh = shfl64(c, (lane + 31) & 31);
  const float my_s = lane == 0 ? so : key_score(sh);
  const int64_t my_j = lane == 0 ? own : key_chunk(sh);
  const bool live = lane < P.k && my_j >= 0 && my_s != -INFINITY;
  float m = live ? my_s : -INFINITY;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, o));
  const float ex = live ? __expf(my_s - m) : 0.f;
  float z = ex;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(kFull, z, o);
  if (lane < P.k) {
    idx[bh * P.k + lane] = live ? (int32_t)my_j : -1;
    w[bh * P.k + lane] = live ? ex / z : 0.f;
  }
}

// The summed outputs in the storage dtype; seq_lens advanced when appending.
__global__ void cp_finish_kernel(Params P, const float* sum, void* out, bool append, int64_t n) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) store_elem(out, P.dtype, i, sum[i]);
  if (append && blockIdx.x == 0)
    for (int b = threadIdx.x; b < P.B; b += blockDim.x) P.seq_lens[b] += 1;
}

int chunks_per_cta(const Params& P) {
  if (P.dtype == HILS_BF16) return P.d == 64 ? Geo<64, 2>::CPS : Geo<128, 2>::CPS;
  return P.d == 64 ? Geo<64, 4>::CPS : Geo<128, 4>::CPS;
}

}  // namespace

static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

size_t decode_ws_bytes(const Params& P, DecodeWs* out, char* base) {
  DecodeWs w{};
  // as few ranges as the CTA geometry allows, then the chunks spread evenly over them
  const int cps_max = chunks_per_cta(P);
  w.n_split = (P.max_chunks + cps_max - 1) / cps_max;
  if (w.n_split < 1) w.n_split = 1;
  w.chunks_per_split = (P.max_chunks + w.n_split - 1) / w.n_split;
  const int K = P.k - 1 > 0 ? P.k - 1 : 1;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    char* p = base ? base + off : nullptr;
    off += align256(bytes);
    return p;
  };
  const int64_t nc = (int64_t)P.B * P.Hq * w.n_split * K;
  w.cand = (uint64_t*)take(sizeof(uint64_t) * nc);
  w.idx = (int32_t*)take(sizeof(int32_t) * P.B * P.Hq * P.k);
  w.w = (float*)take(sizeof(float) * P.B * P.Hq * P.k);
  w.page = (int32_t*)take(sizeof(int32_t) * P.B * P.Hq * P.k);
  w.ticket_bytes = sizeof(int32_t) * ((size_t)P.B * P.Hkv + P.B);
  w.tickets = (int32_t*)take(w.ticket_bytes);
  if (out) *out = w;
  return off;
}

size_t decode_smem_bytes(const Params& P, const DecodeWs& ws) {
  return ScanSmem{P.d, P.r, P.group, chunks_per_cta(P), ws.n_split, P.k}.bytes();
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

cudaError_t launch_cp_candidates(const Params& P, const void* k_new, const void* v_new,
                                 const DecodeWs& ws_in, cudaStream_t s) {
  DecodeWs ws = ws_in;
  ws.append = k_new != nullptr;
  if (P.dtype == HILS_BF16)
    return P.d == 64 ? launch_scan<64, 2>(P, k_new, v_new, ws, nullptr, nullptr, s)
                     : launch_scan<128, 2>(P, k_new, v_new, ws, nullptr, nullptr, s);
  return P.d == 64 ? launch_scan<64, 4>(P, k_new, v_new, ws, nullptr, nullptr, s)
                   : launch_scan<128, 4>(P, k_new, v_new, ws, nullptr, nullptr, s);
}

cudaError_t launch_cp_select(const Params& P, int world, const uint64_t* keys,
                             const float* own_scores, bool append, int32_t* idx, float* w,
                             cudaStream_t s) {
  HILS_PROFILE("decode_cp.select", s);
  cp_select_kernel<<<dim3(P.Hq, P.B), 32, 0, s>>>(P, world, keys, own_scores, append, idx, w);
  return cudaGetLastError();
}

cudaError_t launch_cp_attend(const Params& P, int64_t chunk_base, const void* k_new,
                             const void* v_new, const int32_t* idx, const float* w, float* partial,
                             cudaStream_t s) {
  DecodeWs ws{};   // no workspace: the selection comes from idx and w, the pages from the cache
  ws.idx = const_cast<int32_t*>(idx);
  ws.w = const_cast<float*>(w);
  ws.append = k_new != nullptr;
  ws.chunk_base = chunk_base;
  ws.cp_partial = partial;
  if (P.dtype == HILS_BF16)
    return P.d == 64 ? launch_attend<64, 2>(P, ws, k_new, v_new, nullptr, s)
                     : launch_attend<128, 2>(P, ws, k_new, v_new, nullptr, s);
  return P.d == 64 ? launch_attend<64, 4>(P, ws, k_new, v_new, nullptr, s)
                   : launch_attend<128, 4>(P, ws, k_new, v_new, nullptr, s);
}

cudaError_t launch_cp_finish(const Params& P, const float* sum, void* out, bool append,
                             cudaStream_t s) {
  const int64_t n = (int64_t)P.B * P.Hq * P.d;
  HILS_PROFILE("decode_cp.finish", s);
  const unsigned blocks = (unsigned)((n + 255) / 256 > 0 ? (n + 255) / 256 : 1);
  cp_finish_kernel<<<blocks, 256, 0, s>>>(P, sum, out, append, n);
  return cudaGetLastError();
}

}  // namespace hils
