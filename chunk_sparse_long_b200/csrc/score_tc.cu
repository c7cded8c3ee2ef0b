// Prefill calibration, landmark scoring, selection and fusion weights (a1-a4)
// with the landmark GEMM on the 5th-generation tensor cores.
//
// CTA = 128 consecutive query positions of one (sequence, query head); thread
// t owns row t, which is also TMEM lane t.
//
//   a1  thread t computes q~ = q + (qA)B in float32 and splits it into three
//       bf16 terms hi + mid + lo (each the bf16 rounding of what is left), so
//       q~ - (hi + mid + lo) is below 2^-27 |q~|; the three terms are written
//       as three 128-row K-major swizzled tiles.
//   a2  for every block of 128 causally visible chunks of the row's KV head:
//       the landmark block is copied into shared memory (double-buffered,
//       prefetched one block ahead) and S = sum over terms of Q_term LM^T is
//       accumulated by 3 x d/16 tcgen05.mma (M=128, N=128) into one of two
//       TMEM buffers, so the MMAs of block n+1 run while block n is consumed.
//   a3  thread t reads its 128 scores from TMEM, 32 columns at a time, and keeps
//       the k-1 best candidates j < own in a sorted list held in registers
//       (worst kept entry first).  A lane first builds the bitmask of columns
//       that beat its worst entry (the same work in every lane), then the warp
//       loops max(popcount) times, each lane inserting its next set column
//       through an unrolled compare-and-shift network -- lanes do not
//       serialise each other's inserts and nothing waits on memory.  Strict
//       '>' against the worst entry while j ascends keeps the lower index on
//       ties; the own chunk's score is kept apart.
//   a4  softmax of the own and selected scores -> idx, w.
#include <cfloat>

#include "hils_common.cuh"
#include "tc_common.cuh"

namespace hils {
namespace {

constexpr int kRowsS = 128;     // query rows per CTA (M)
constexpr int kBlk = 128;       // landmark chunks per block (N)
constexpr int kThrS = 128;
constexpr int kTerms = 3;
constexpr uint32_t kTmemColsS = 256;  // two S buffers of 128 columns
constexpr int kLmBufs = 3;            // landmark blocks in flight: prefetch distance 2
constexpr int kBulkPasses = 12;       // a chunk this dense for some lane is merged in bulk

template <int D>
struct ScoreLayout {
  static constexpr uint32_t kQt = kRowsS * D * 2;             // one q~ term tile
  static constexpr uint32_t kLmB = kBlk * D * 2;              // one landmark block
  static constexpr uint32_t kQ = 0;                           // kTerms tiles
  static constexpr uint32_t kLm = kTerms * kQt;               // kLmBufs blocks
  static constexpr uint32_t kScratch = kLm + kLmBufs * kLmB;  // calibration t = qA [r][128]
  static constexpr uint32_t kEnd = kScratch + kMaxRank * kThrS * 4;
  static constexpr uint32_t kSmem = kEnd + 1024;
};

// Landmark block `blk` (chunks blk*128 ..) of (b, g) into swizzled K-major tile at lm_smem.
template <int D>
__device__ __forceinline__ void load_lm_block(const Params& P, uint32_t lm_smem, int b, int g,
                                              int64_t blk, int64_t last_chunk, int tid) {
  const uint16_t* base = reinterpret_cast<const uint16_t*>(P.landmarks);
  for (int x = tid; x < kBlk * (D / 8); x += kThrS) {
    const int rr = x / (D / 8), c = x % (D / 8);
    const int64_t j = blk * kBlk + rr;
    const bool in = j <= last_chunk;
    const uint16_t* src = base + ((((int64_t)b * P.max_chunks + (in ? j : 0)) * P.Hkv + g) * D + c * 8);
    tc::cp_async16(lm_smem + (uint32_t)(c >> 3) * (kBlk * 128) + tc::swz(rr, c & 7), src,
                   in ? 16u : 0u);
  }
}

// (sa, ja) ranks below (sb, jb) in the (score desc, index asc) order.
__device__ __forceinline__ bool worse(float sa, int ja, float sb, int jb) {
  return sa < sb || (sa == sb && ja > jb);
}

// The k-1 best candidates of one row, kept in registers in ascending order
// (index 0 = the worst kept entry, compared against every new candidate).
// Slots [K, KS) hold +inf sentinels that no candidate beats, slots [0, K)
// start as -inf sentinels that every candidate beats; KS is a compile-time
// bound so the insertion network below is fully unrolled (no local memory).
template <int KS>
struct RegList {
  float s[KS];
  int j[KS];

  __device__ __forceinline__ void init(int K) {
#pragma unroll
    for (int p = 0; p < KS; ++p) {
      s[p] = p < K ? -INFINITY : INFINITY;
      j[p] = p < K ? INT32_MAX : -1;
    }
  }
  // Drops entry 0 and inserts (ns, nj), which must rank above entry 0.  New
  // candidates arrive in ascending chunk order, so a kept entry with the same
  // score always ranks above the new one: comparing scores alone decides.
  // Every slot takes its upper neighbour, the new entry, or keeps its value.
  __device__ __forceinline__ void insert(float ns, int nj) {
    bool c[KS + 1];
#pragma unroll
    for (int p = 0; p < KS; ++p) c[p] = s[p] < ns;
    c[KS] = false;
#pragma unroll
    for (int p = 0; p < KS; ++p) {
      const bool up = p + 1 < KS && c[p + 1];
      s[p] = up ? s[p + 1] : (c[p] ? ns : s[p]);
      j[p] = up ? j[p + 1] : (c[p] ? nj : j[p]);
    }
  }
  // Merges 32 new candidates (any order; masked ones as (-inf, INT32_MAX)) into
  // the list: bitonic sort of the 32 (worst first), then the best KS of the
  // union by one bitonic merge.  The +inf sentinels above slot K are the best
  // of all, so exactly the best K real entries stay in slots [0, K).
  __device__ __forceinline__ void merge32(float (&vs)[32], int (&vj)[32]) {
#pragma unroll
    for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
      for (int m = k >> 1; m > 0; m >>= 1) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int l = i ^ m;
          if (l > i) {
            const bool up = (i & k) == 0;          // ascending block: worst first
            const bool swap = up ? worse(vs[l], vj[l], vs[i], vj[i])
                                 : worse(vs[i], vj[i], vs[l], vj[l]);
            if (swap) {
              const float ts = vs[i]; vs[i] = vs[l]; vs[l] = ts;
              const int tj = vj[i]; vj[i] = vj[l]; vj[l] = tj;
            }
          }
        }
      }
    }
    // best KS of the list (ascending) and the top KS of vs (ascending): slot p
    // takes the better of s[p] and the (p+1)-th best of vs, which leaves a
    // bitonic sequence holding the best KS; a bitonic merge sorts it
#pragma unroll
    for (int p = 0; p < KS; ++p) {
      const float cs = vs[32 - KS + (KS - 1 - p)];
      const int cj = vj[32 - KS + (KS - 1 - p)];
      if (worse(s[p], j[p], cs, cj)) {
        s[p] = cs;
        j[p] = cj;
      }
    }
#pragma unroll
    for (int m = KS >> 1; m > 0; m >>= 1) {
#pragma unroll
      for (int i = 0; i < KS; ++i) {
        const int l = i ^ m;
        if (l > i && worse(s[l], j[l], s[i], j[i])) {
          const float ts = s[i]; s[i] = s[l]; s[l] = ts;
          const int tj = j[i]; j[i] = j[l]; j[l] = tj;
        }
      }
    }
  }
};

// v[x] for a runtime x in 0..31 without dynamic register indexing (select tree).
__device__ __forceinline__ uint32_t pick32(const uint32_t (&v)[32], int x) {
  uint32_t a[16];
#pragma unroll
  for (int u = 0; u < 16; ++u) a[u] = (x & 16) ? v[u + 16] : v[u];
#pragma unroll
  for (int u = 0; u < 8; ++u) a[u] = (x & 8) ? a[u + 8] : a[u];
#pragma unroll
  for (int u = 0; u < 4; ++u) a[u] = (x & 4) ? a[u + 4] : a[u];
#pragma unroll
  for (int u = 0; u < 2; ++u) a[u] = (x & 2) ? a[u + 2] : a[u];
  return (x & 1) ? a[1] : a[0];
}

template <int D, int KS>
__global__ void __launch_bounds__(kThrS, 1) score_tc_kernel(Params P, int32_t* idx, float* w) {
  using Lay = ScoreLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bar[2];
  __shared__ uint32_t tmem_sh;
  __shared__ int abort_sh;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~(uintptr_t)1023);
  const uint32_t sbase = tc::smem_u32(smem);
  const int tid = threadIdx.x, warp = tid >> 5;
  const int h = blockIdx.y, b = blockIdx.z;
  const int g = h / P.group;
  const int64_t i = (int64_t)blockIdx.x * kRowsS + tid;
  const bool valid = i < P.L;
  const int64_t pos = P.pos0 + (valid ? i : P.L - 1);
  const int64_t own = pos / kChunk;
  const int64_t r = ((int64_t)b * P.L + i) * P.Hq + h;
  const int64_t i_last = min((int64_t)(blockIdx.x + 1) * kRowsS, P.L) - 1;
  const int64_t own_max = (P.pos0 + i_last) / kChunk;
  const int n_blk = (int)(own_max / kBlk) + 1;

  if (tid == 0) {
    tc::mbar_init(&bar[0], 1);
    tc::mbar_init(&bar[1], 1);
    tc::fence_mbar_init();
    abort_sh = 0;
  }
  if (warp == 0) {
    tc::tmem_alloc(&tmem_sh, kTmemColsS);
    tc::tmem_relinquish();
  }

  // ---- a1: q~ in float32 (A, B staged in the landmark buffers, qA in scratch) --
  float qt[D];
#pragma unroll
  for (int e = 0; e < D; e += 8) {
    if (valid) {
      load8(P.q, HILS_BF16, r * D + e, &qt[e]);
    } else {
#pragma unroll
      for (int u = 0; u < 8; ++u) qt[e + u] = 0.f;
    }
  }
  if (P.r > 0) {
    const int r4 = (P.r + 3) & ~3;                 // A rows padded to a multiple of 4
    float* sA = reinterpret_cast<float*>(smem + Lay::kLm);        // [D][r4]
    float* sB = sA + D * r4;                                      // [r][D]
    float* sT = reinterpret_cast<float*>(smem + Lay::kScratch);   // [r4][128]
    for (int x = tid; x < D * r4; x += kThrS) {
      const int e = x / r4, a = x % r4;
      sA[x] = a < P.r ? P.A[e * P.r + a] : 0.f;
    }
    for (int x = tid; x < P.r * D; x += kThrS) sB[x] = P.Bm[x];
    __syncthreads();
    // t = q A: four independent accumulator chains per pass, 16-byte broadcast loads
    for (int a = 0; a < r4; a += 4) {
      float t0 = 0.f, t1 = 0.f, t2 = 0.f, t3 = 0.f;
#pragma unroll
      for (int e = 0; e < D; ++e) {
        const float4 av = *reinterpret_cast<const float4*>(sA + e * r4 + a);
        t0 = fmaf(qt[e], av.x, t0);
        t1 = fmaf(qt[e], av.y, t1);
        t2 = fmaf(qt[e], av.z, t2);
        t3 = fmaf(qt[e], av.w, t3);
      }
      sT[(a + 0) * kThrS + tid] = t0;
      sT[(a + 1) * kThrS + tid] = t1;
      sT[(a + 2) * kThrS + tid] = t2;
      sT[(a + 3) * kThrS + tid] = t3;
    }
    // q~ = q + t B
    for (int a = 0; a < P.r; ++a) {
      const float ta = sT[a * kThrS + tid];
#pragma unroll
      for (int e = 0; e < D; e += 4) {
        const float4 bv = *reinterpret_cast<const float4*>(sB + a * D + e);
        qt[e] = fmaf(ta, bv.x, qt[e]);
        qt[e + 1] = fmaf(ta, bv.y, qt[e + 1]);
        qt[e + 2] = fmaf(ta, bv.z, qt[e + 2]);
        qt[e + 3] = fmaf(ta, bv.w, qt[e + 3]);
      }
    }
  }
  // three-term bf16 split of q~ into the A tiles
#pragma unroll
  for (int c = 0; c < D / 8; ++c) {
    uint32_t hw[4], mw[4], lw[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      float x0 = qt[c * 8 + 2 * u], x1 = qt[c * 8 + 2 * u + 1];
      hw[u] = tc::pack_bf16x2(x0, x1);
      x0 -= __uint_as_float(hw[u] << 16);
      x1 -= __uint_as_float(hw[u] & 0xFFFF0000u);
      mw[u] = tc::pack_bf16x2(x0, x1);
      x0 -= __uint_as_float(mw[u] << 16);
      x1 -= __uint_as_float(mw[u] & 0xFFFF0000u);
      lw[u] = tc::pack_bf16x2(x0, x1);
    }
    const uint32_t off = (uint32_t)(c >> 3) * (kRowsS * 128) + tc::swz(tid, c & 7);
    *reinterpret_cast<uint4*>(smem + Lay::kQ + 0 * Lay::kQt + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    *reinterpret_cast<uint4*>(smem + Lay::kQ + 1 * Lay::kQt + off) = make_uint4(mw[0], mw[1], mw[2], mw[3]);
    *reinterpret_cast<uint4*>(smem + Lay::kQ + 2 * Lay::kQt + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
  }
  tc::fence_proxy_async();
  tc::tc_fence_before();
  __syncthreads();   // A, B and t scratch are dead from here on
  tc::tc_fence_after();
  const uint32_t tmem = tmem_sh;
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
  constexpr uint32_t kId = tc::idesc_bf16(kRowsS, kBlk, 0);

  // ---- a2/a3: landmark blocks --------------------------------------------
  const int K = P.k - 1;
  RegList<KS> list;
  list.init(K);
  float s_own = 0.f;
  uint32_t phase[2] = {0u, 0u};

  // landmark blocks 0 and 1 up front; block b+2 is issued while block b is consumed
  load_lm_block<D>(P, sbase + Lay::kLm, b, g, 0, own_max, tid);
  if (n_blk > 1) load_lm_block<D>(P, sbase + Lay::kLm + Lay::kLmB, b, g, 1, own_max, tid);
  tc::cp_async_commit();

  auto consume = [&](int blk) {
    const int sb = blk & 1;
    if (!tc::mbar_wait(&bar[sb], phase[sb])) abort_sh = 1;
    phase[sb] ^= 1;
    tc::tc_fence_after();
    const int64_t j0 = (int64_t)blk * kBlk;
#pragma unroll 1
    for (int c0 = 0; c0 < kBlk; c0 += 32) {
      // tcgen05.ld is warp-collective: every lane loads all columns
      uint32_t sv[32];
      tc::tmem_ld32(tmem + sb * kBlk + lane_off + c0, sv);
      tc::tmem_ld_wait();
      uint32_t m = 0;
      const float thr = list.s[0];
#pragma unroll
      for (int x = 0; x < 32; ++x) {
        const int64_t j = j0 + c0 + x;
        const float s = __uint_as_float(sv[x]) * P.inv_sqrt_d;
        if (j == own) s_own = s;
        m |= (j < own && s > thr) ? (1u << x) : 0u;
      }
      if (__reduce_max_sync(0xffffffffu, (unsigned)__popc(m)) >= kBulkPasses) {
        // dense chunk: sort the 32 columns and merge them in one go
        float vs[32];
        int vj[32];
#pragma unroll
        for (int x = 0; x < 32; ++x) {
          const bool in = (m >> x) & 1u;
          vs[x] = in ? __uint_as_float(sv[x]) * P.inv_sqrt_d : -INFINITY;
          vj[x] = in ? (int)(j0 + c0 + x) : INT32_MAX;
        }
        list.merge32(vs, vj);
        m = 0;
      }
      while (__any_sync(0xffffffffu, m != 0)) {
        if (m) {
          const int x = __ffs(m) - 1;
          m &= m - 1;
          const float s = __uint_as_float(pick32(sv, x)) * P.inv_sqrt_d;
          if (s > list.s[0]) list.insert(s, (int)(j0 + c0 + x));
        }
      }
    }
  };

  for (int blk = 0; blk < n_blk; ++blk) {
    const int sb = blk & 1;
    const uint32_t lm = sbase + Lay::kLm + (blk % kLmBufs) * Lay::kLmB;
    // landmark block blk has landed (issued two blocks earlier, or up front)
    if (blk + 1 < n_blk && blk > 0) tc::cp_async_wait<1>(); else tc::cp_async_wait<0>();
    tc::fence_proxy_async();
    tc::tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc::tc_fence_after();
#pragma unroll
      for (int term = 0; term < kTerms; ++term) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t a = tc::smem_desc(sbase + Lay::kQ + term * Lay::kQt +
                                               (kk >> 2) * (kRowsS * 128) + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = tc::smem_desc(lm + (kk >> 2) * (kBlk * 128) + (kk & 3) * 32, 16, 1024);
          tc::mma_bf16(tmem + sb * kBlk, a, bd, kId, (term | kk) != 0);
        }
      }
      tc::mma_commit(&bar[sb]);
    }
    if (blk > 0) {
      consume(blk - 1);
      // the MMAs of block blk-1 are done: its landmark buffer takes block blk+2
      if (blk + 2 < n_blk) {
        load_lm_block<D>(P, sbase + Lay::kLm + ((blk + 2) % kLmBufs) * Lay::kLmB, b, g, blk + 2,
                         own_max, tid);
        tc::cp_async_commit();
      }
    } else if (n_blk > 2) {
      load_lm_block<D>(P, sbase + Lay::kLm + (2 % kLmBufs) * Lay::kLmB, b, g, 2, own_max, tid);
      tc::cp_async_commit();
    }
  }
  consume(n_blk - 1);

  // ---- a4: fusion weights; the list is read best-first -------------------
  if (valid) {
    float m = s_own;
#pragma unroll
    for (int p = 0; p < KS; ++p)
      if (list.j[p] != INT32_MAX && list.j[p] >= 0) m = fmaxf(m, list.s[p]);
    float z = __expf(s_own - m);
#pragma unroll
    for (int p = 0; p < KS; ++p)
      if (list.j[p] != INT32_MAX && list.j[p] >= 0) z += __expf(list.s[p] - m);
    const float iz = 1.f / z;
    int32_t* ix = idx + r * P.k;
    float* wr = w + r * P.k;
    ix[0] = (int32_t)own;
    wr[0] = __expf(s_own - m) * iz;
    int n = 1;
#pragma unroll
    for (int p = KS - 1; p >= 0; --p) {
      if (list.j[p] != INT32_MAX && list.j[p] >= 0) {
        ix[n] = list.j[p];
        wr[n] = __expf(list.s[p] - m) * iz;
        ++n;
      }
    }
    for (int a = n; a < P.k; ++a) {
      ix[a] = -1;
      wr[a] = 0.f;
    }
  }
  if (abort_sh && tid == 0) set_device_error(kErrTimeout);
  tc::cp_async_wait<0>();
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, kTmemColsS);
}

template <int D, int KS>
cudaError_t run_score_tc(const Params& P, int32_t* idx, float* w, cudaStream_t s) {
  using Lay = ScoreLayout<D>;
  cudaError_t e = cudaFuncSetAttribute(score_tc_kernel<D, KS>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Lay::kSmem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)((P.L + kRowsS - 1) / kRowsS), P.Hq, P.B);
  HILS_PROFILE("prefill.select_tc", s);
  score_tc_kernel<D, KS><<<grid, kThrS, Lay::kSmem, s>>>(P, idx, w);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_select_tc(const Params& P, int32_t* idx, float* w, cudaStream_t s) {
  // the register list holds 16 or 32 slots (k-1 <= 31)
  if (P.k - 1 <= 16)
    return P.d == 64 ? run_score_tc<64, 16>(P, idx, w, s) : run_score_tc<128, 16>(P, idx, w, s);
  return P.d == 64 ? run_score_tc<64, 32>(P, idx, w, s) : run_score_tc<128, 32>(P, idx, w, s);
}

}  // namespace hils
