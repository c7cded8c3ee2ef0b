// Prefill calibration, landmark scoring, selection and fusion weights (a1-a4)
// for bf16 inputs, as three kernels that each run at the occupancy their work
// wants:
//
//   calib_kernel (a1)   one thread per query row computes q~ = q + (qA)B in
//       float32 and splits it into three bf16 terms hi + mid + lo (each the
//       bf16 rounding of what is left, so q~ - (hi + mid + lo) is below
//       2^-27 |q~|).  The terms are written as ready-made shared-memory
//       images: per 128-row tile, three K-major 128-byte-swizzled tiles.
//   score_tc_kernel (a2)  persistent; per 128-row tile one bulk copy brings
//       the three term tiles in, and for every block of 128 causally visible
//       chunks S = sum over terms Q_term LM^T runs as 3 x d/16 tcgen05.mma
//       (M = N = 128, float32 accumulate) into one of two TMEM buffers while
//       the previous block is read back and streamed out as scaled float32
//       scores.  Landmark blocks are prefetched two steps ahead, across tile
//       boundaries too.
//   select_kernel (a3, a4)  one thread per row keeps the k-1 best candidates
//       j < own in a min-heap of 64-bit keys in shared memory (root = the
//       worst kept entry), reading its scores 32 columns at a time; candidates
//       that beat the root are inserted one set bit at a time across the
//       warp, so lanes do not serialise each other's inserts.  Strict '>'
//       against the root while j ascends keeps the lower index on ties.  A
//       heap sort then yields the list best-first, and the softmax of the
//       own and selected scores gives the weights.
//
// Score workspace layout: per (sequence, head), the tiles of 128 rows in
// order; tile t holds score_tile_blocks(t) * 128 columns (the blocks of chunks
// its rows can see) as [column / 4][128 rows][4] float32, so a warp reads or
// writes 512 contiguous bytes per 16-byte access.
#include <cfloat>

#include "hils_common.cuh"
#include "tc_common.cuh"

namespace hils {
namespace {

constexpr int kRowsS = kScoreTileRows;  // query rows per tile (M)
constexpr int kBlk = kScoreBlock;       // landmark chunks per block (N)
constexpr int kThrS = 128;
constexpr int kTerms = 3;
constexpr uint32_t kTmemColsS = 256;  // two S buffers of 128 columns
constexpr int kLmBufs = 3;            // landmark blocks in flight: prefetch distance 2

template <int D>
struct ScoreLayout {
  static constexpr uint32_t kQt = kRowsS * D * 2;             // one q~ term tile
  static constexpr uint32_t kQimg = kTerms * kQt;             // one tile's three terms
  static constexpr uint32_t kLmB = kBlk * D * 2;              // one landmark block
  static constexpr uint32_t kQ = 0;
  static constexpr uint32_t kLm = kQimg;                      // kLmBufs blocks
  static constexpr uint32_t kEnd = kLm + kLmBufs * kLmB;
  static constexpr uint32_t kSmem = kEnd + 1024;
};

// ---- a1: calibration ------------------------------------------------------
// RP = calibration rank rounded up (A staged as [D][RP] with zero columns).
// Each thread computes NR rows (row tid of NR consecutive tiles), so every
// 16-byte broadcast load of A or B feeds NR x 4 FMAs.
template <int D, int RP, int NR>
__global__ void __launch_bounds__(kThrS) calib_kernel(Params P, uint8_t* qimg, int T,
                                                      int64_t n_tiles) {
  using Lay = ScoreLayout<D>;
  extern __shared__ float smf[];
  float* sA = smf;            // [D][RP]
  float* sB = smf + D * RP;   // [RP][D]
  const int tid = threadIdx.x;
  for (int x = tid; x < D * RP; x += kThrS) {
    const int e = x / RP, a = x % RP;
    sA[x] = a < P.r ? P.A[e * P.r + a] : 0.f;
  }
  for (int x = tid; x < RP * D; x += kThrS) sB[x] = x < P.r * D ? P.Bm[x] : 0.f;
  __syncthreads();

  const int64_t n_groups = (n_tiles + NR - 1) / NR;
  for (int64_t gg = blockIdx.x; gg < n_groups; gg += gridDim.x) {
    int64_t qoff[NR];
    bool valid[NR];
#pragma unroll
    for (int v = 0; v < NR; ++v) {
      const int64_t g = gg * NR + v;
      const int t = (int)(g % T);
      const int64_t bh = g / T;
      const int h = (int)(bh % P.Hq), b = (int)(bh / P.Hq);
      const int64_t i = (int64_t)t * kRowsS + tid;
      valid[v] = g < n_tiles && i < P.L;
      qoff[v] = valid[v] ? (((int64_t)b * P.L + i) * P.Hq + h) * D : 0;
    }
    // t = q A: one accumulator chain per rank column, summed over e in order
    float ta[NR][RP];
#pragma unroll
    for (int v = 0; v < NR; ++v)
#pragma unroll
      for (int a = 0; a < RP; ++a) ta[v][a] = 0.f;
    if (P.r > 0) {
#pragma unroll 1
      for (int e0 = 0; e0 < D; e0 += 8) {
        float qv[NR][8];
#pragma unroll
        for (int v = 0; v < NR; ++v) {
          if (valid[v]) {
            load8(P.q, HILS_BF16, qoff[v] + e0, qv[v]);
          } else {
#pragma unroll
            for (int u = 0; u < 8; ++u) qv[v][u] = 0.f;
          }
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
#pragma unroll
          for (int a = 0; a < RP; a += 4) {
            const float4 av = *reinterpret_cast<const float4*>(sA + (e0 + u) * RP + a);
#pragma unroll
            for (int v = 0; v < NR; ++v) {
              ta[v][a] = fmaf(qv[v][u], av.x, ta[v][a]);
              ta[v][a + 1] = fmaf(qv[v][u], av.y, ta[v][a + 1]);
              ta[v][a + 2] = fmaf(qv[v][u], av.z, ta[v][a + 2]);
              ta[v][a + 3] = fmaf(qv[v][u], av.w, ta[v][a + 3]);
            }
          }
        }
      }
    }
    // q~ = q + t B (a ascending), then the three-term split, 8 elements at a time
#pragma unroll 1
    for (int c = 0; c < D / 8; ++c) {
      float x[NR][8];
#pragma unroll
      for (int v = 0; v < NR; ++v) {
        if (valid[v]) {
          load8(P.q, HILS_BF16, qoff[v] + c * 8, x[v]);
        } else {
#pragma unroll
          for (int u = 0; u < 8; ++u) x[v][u] = 0.f;
        }
      }
#pragma unroll
      for (int a = 0; a < RP; ++a) {
        if (a < P.r) {
          const float4 b0 = *reinterpret_cast<const float4*>(sB + a * D + c * 8);
          const float4 b1 = *reinterpret_cast<const float4*>(sB + a * D + c * 8 + 4);
#pragma unroll
          for (int v = 0; v < NR; ++v) {
            x[v][0] = fmaf(ta[v][a], b0.x, x[v][0]);
            x[v][1] = fmaf(ta[v][a], b0.y, x[v][1]);
            x[v][2] = fmaf(ta[v][a], b0.z, x[v][2]);
            x[v][3] = fmaf(ta[v][a], b0.w, x[v][3]);
            x[v][4] = fmaf(ta[v][a], b1.x, x[v][4]);
            x[v][5] = fmaf(ta[v][a], b1.y, x[v][5]);
            x[v][6] = fmaf(ta[v][a], b1.z, x[v][6]);
            x[v][7] = fmaf(ta[v][a], b1.w, x[v][7]);
          }
        }
      }
      const uint32_t off = (uint32_t)(c >> 3) * (kRowsS * 128) + tc::swz(tid, c & 7);
#pragma unroll
      for (int v = 0; v < NR; ++v) {
        if (gg * NR + v >= n_tiles) continue;
        uint32_t hw[4], mw[4], lw[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          float x0 = x[v][2 * u], x1 = x[v][2 * u + 1];
          hw[u] = tc::pack_bf16x2(x0, x1);
          x0 -= __uint_as_float(hw[u] << 16);
          x1 -= __uint_as_float(hw[u] & 0xFFFF0000u);
          mw[u] = tc::pack_bf16x2(x0, x1);
          x0 -= __uint_as_float(mw[u] << 16);
          x1 -= __uint_as_float(mw[u] & 0xFFFF0000u);
          lw[u] = tc::pack_bf16x2(x0, x1);
        }
        uint8_t* img = qimg + (gg * NR + v) * Lay::kQimg;
        *reinterpret_cast<uint4*>(img + 0 * Lay::kQt + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
        *reinterpret_cast<uint4*>(img + 1 * Lay::kQt + off) = make_uint4(mw[0], mw[1], mw[2], mw[3]);
        *reinterpret_cast<uint4*>(img + 2 * Lay::kQt + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
      }
    }
  }
}

// ---- a2: landmark scores on the tensor cores --------------------------------
// Landmark block `blk` (chunks blk*128 ..) of (b, g) into a swizzled K-major tile.
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

// One (tile, landmark block) step of a CTA's walk over its tiles.
struct Step {
  int64_t g;   // tile id ((b * Hq + h) * T + t); >= n_tiles once the walk is over
  int blk, nblk;
};

__device__ __forceinline__ void step_set(Step& s, int64_t g, const Params& P, int T,
                                         int64_t n_tiles) {
  s.g = g;
  s.blk = 0;
  s.nblk = g < n_tiles ? (int)score_tile_blocks(P.L, P.pos0, (int)(g % T)) : 0;
}

__device__ __forceinline__ void step_next(Step& s, const Params& P, int T, int64_t n_tiles) {
  if (++s.blk >= s.nblk) step_set(s, s.g + gridDim.x, P, T, n_tiles);
}

template <int D>
__device__ __forceinline__ void load_lm_step(const Params& P, uint32_t lm_smem, const Step& s,
                                             int T, int tid) {
  const int t = (int)(s.g % T);
  const int64_t bh = s.g / T;
  const int b = (int)(bh / P.Hq), g = (int)(bh % P.Hq) / P.group;
  const int64_t last = min((int64_t)(t + 1) * kRowsS, P.L) - 1;
  load_lm_block<D>(P, lm_smem, b, g, s.blk, (P.pos0 + last) / kChunk, tid);
}

template <int D>
__global__ void __launch_bounds__(kThrS, 1) score_tc_kernel(Params P, const uint8_t* qimg,
                                                           float* scores, int T, int64_t n_tiles,
                                                           int64_t cols_per_head) {
  using Lay = ScoreLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bar[2];   // MMAs into S buffer 0 / 1 done
  __shared__ uint64_t qbar;     // q~ terms of the current tile landed
  __shared__ uint32_t tmem_sh;
  __shared__ int abort_sh;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~(uintptr_t)1023);
  const uint32_t sbase = tc::smem_u32(smem);
  const int tid = threadIdx.x, warp = tid >> 5;
  if ((int64_t)blockIdx.x >= n_tiles) return;

  if (tid == 0) {
    tc::mbar_init(&bar[0], 1);
    tc::mbar_init(&bar[1], 1);
    tc::mbar_init(&qbar, 1);
    tc::fence_mbar_init();
    abort_sh = 0;
  }
  if (warp == 0) {
    tc::tmem_alloc(&tmem_sh, kTmemColsS);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = tmem_sh;
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
  constexpr uint32_t kId = tc::idesc_bf16(kRowsS, kBlk, 0);

  auto load_q = [&](int64_t g) {
    tc::mbar_arrive_expect_tx(&qbar, Lay::kQimg);
#pragma unroll
    for (int term = 0; term < kTerms; ++term)
      tc::bulk_g2s(sbase + Lay::kQ + term * Lay::kQt, qimg + g * Lay::kQimg + term * Lay::kQt,
                   Lay::kQt, &qbar);
  };

  Step cur, pf;
  step_set(cur, blockIdx.x, P, T, n_tiles);
  pf = cur;
  // landmark blocks of the first two steps; exactly one cp.async group per step
  load_lm_step<D>(P, sbase + Lay::kLm, pf, T, tid);
  tc::cp_async_commit();
  step_next(pf, P, T, n_tiles);
  if (pf.g < n_tiles) {
    load_lm_step<D>(P, sbase + Lay::kLm + Lay::kLmB, pf, T, tid);
    step_next(pf, P, T, n_tiles);
  }
  tc::cp_async_commit();
  if (tid == 0) load_q(cur.g);

  uint32_t phase[2] = {0u, 0u}, qphase = 0u;
  Step prev = cur;   // the step whose scores are drained next
  int64_t n = 0;     // steps issued so far

  auto wait_mma = [&](int64_t sidx) {
    const int sb = (int)(sidx & 1);
    if (!tc::mbar_wait(&bar[sb], phase[sb])) abort_sh = 1;
    phase[sb] ^= 1;
    tc::tc_fence_after();
  };
  // S buffer of step sidx -> scaled scores of tile st.g, columns st.blk * 128 ..
  auto drain = [&](int64_t sidx, const Step& st) {
    const int sb = (int)(sidx & 1);
    const int t = (int)(st.g % T);
    const int64_t bh = st.g / T;
    float4* dst = reinterpret_cast<float4*>(
        scores + (bh * cols_per_head + score_tile_cols_before(P.L, P.pos0, t) +
                  (int64_t)st.blk * kBlk) * kRowsS);
#pragma unroll 1
    for (int c0 = 0; c0 < kBlk; c0 += 32) {
      uint32_t sv[32];
      tc::tmem_ld32(tmem + sb * kBlk + lane_off + c0, sv);
      tc::tmem_ld_wait();
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        float4 v;
        v.x = __uint_as_float(sv[4 * u]) * P.inv_sqrt_d;
        v.y = __uint_as_float(sv[4 * u + 1]) * P.inv_sqrt_d;
        v.z = __uint_as_float(sv[4 * u + 2]) * P.inv_sqrt_d;
        v.w = __uint_as_float(sv[4 * u + 3]) * P.inv_sqrt_d;
        __stcs(dst + ((c0 >> 2) + u) * kRowsS + tid, v);
      }
    }
  };

  while (cur.g < n_tiles) {
    bool drained = false;
    if (cur.blk == 0 && n > 0) {
      // new tile: the previous tile's MMAs must finish before its q~ terms are replaced
      wait_mma(n - 1);
      if (tid == 0) load_q(cur.g);
      drain(n - 1, prev);
      drained = true;
    }
    // groups committed so far: steps 0 .. n+1; the one of step n must be complete
    tc::cp_async_wait<1>();
    tc::fence_proxy_async();
    tc::tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      if (cur.blk == 0) {
        if (!tc::mbar_wait(&qbar, qphase)) abort_sh = 1;
        qphase ^= 1;
      }
      tc::tc_fence_after();
      const int sb = (int)(n & 1);
      const uint32_t lm = sbase + Lay::kLm + (uint32_t)(n % kLmBufs) * Lay::kLmB;
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
    if (n > 0 && !drained) {
      wait_mma(n - 1);
      drain(n - 1, prev);
    }
    // the landmark buffer of step n-1 is free (its MMAs are done): step n+2 goes there
    if (pf.g < n_tiles) {
      load_lm_step<D>(P, sbase + Lay::kLm + (uint32_t)((n + 2) % kLmBufs) * Lay::kLmB, pf, T, tid);
      step_next(pf, P, T, n_tiles);
    }
    tc::cp_async_commit();
    prev = cur;
    step_next(cur, P, T, n_tiles);
    ++n;
  }
  wait_mma(n - 1);
  drain(n - 1, prev);

  if (abort_sh && tid == 0) set_device_error(kErrTimeout);
  tc::cp_async_wait<0>();
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, kTmemColsS);
}

// ---- a3/a4: selection and fusion weights -----------------------------------
// Heap keys: a larger key ranks higher in (score desc, index asc).  The high
// word is the score's bits mapped to an unsigned order (-0 taken as +0), the
// low word is ~j.  Key 0 is an empty slot, below every real entry.
__device__ __forceinline__ uint64_t make_key(float s, int j) {
  uint32_t u = __float_as_uint(s + 0.f);
  u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return ((uint64_t)u << 32) | (uint32_t)(0xFFFFFFFFu - (uint32_t)j);
}
__device__ __forceinline__ float key_score(uint64_t key) {
  if (key == 0) return -INFINITY;
  const uint32_t u = (uint32_t)(key >> 32);
  return __uint_as_float((u & 0x80000000u) ? (u & 0x7FFFFFFFu) : ~u);
}
__device__ __forceinline__ int key_index(uint64_t key) {
  return (int)(0xFFFFFFFFu - (uint32_t)key);
}

// Places x at the root of the min-heap H[0 .. size) (stride kThrS) and sifts it down.
__device__ __forceinline__ void sift_root(uint64_t* H, int size, uint64_t x) {
  int p = 0;
  for (;;) {
    int c = 2 * p + 1;
    if (c >= size) break;
    uint64_t kc = H[c * kThrS];
    if (c + 1 < size) {
      const uint64_t k2 = H[(c + 1) * kThrS];
      if (k2 < kc) {
        kc = k2;
        ++c;
      }
    }
    if (kc >= x) break;
    H[p * kThrS] = kc;
    p = c;
  }
  H[p * kThrS] = x;
}

// v[x] for a runtime x in 0..31 without dynamic register indexing (select tree).
__device__ __forceinline__ float pick32(const float (&v)[32], int x) {
  float a[16];
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

__global__ void __launch_bounds__(kThrS, 6) select_kernel(Params P, const float* scores, int T,
                                                       int64_t cols_per_head, int32_t* idx,
                                                       float* w) {
  extern __shared__ uint64_t heap_sh[];   // [k-1][kThrS]
  const int tid = threadIdx.x;
  const int64_t gtile = blockIdx.x;
  const int t = (int)(gtile % T);
  const int64_t bh = gtile / T;
  const int h = (int)(bh % P.Hq), b = (int)(bh / P.Hq);
  const int64_t i = (int64_t)t * kRowsS + tid;
  const bool valid = i < P.L;
  const int64_t own = valid ? (P.pos0 + i) / kChunk : 0;
  const int64_t i_last = min((int64_t)(t + 1) * kRowsS, P.L) - 1;
  const int64_t own_max = (P.pos0 + i_last) / kChunk;
  const float* St = scores + (bh * cols_per_head + score_tile_cols_before(P.L, P.pos0, t)) * kRowsS;
  const float4* S4 = reinterpret_cast<const float4*>(St);
  const int K = P.k - 1;
  uint64_t* H = heap_sh + tid;
  for (int p = 0; p < K; ++p) H[p * kThrS] = 0;
  float thr = -INFINITY;   // score of the root (the worst kept entry)

  // candidates j < own <= own_max; the tile holds at least own_max + 1 columns
  const int64_t n_scan = K > 0 ? own_max : 0;
#pragma unroll 1
  for (int64_t c0 = 0; c0 < n_scan; c0 += 32) {
    float v[32];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const float4 x = __ldcs(S4 + ((c0 >> 2) + u) * kRowsS + tid);
      v[4 * u] = x.x;
      v[4 * u + 1] = x.y;
      v[4 * u + 2] = x.z;
      v[4 * u + 3] = x.w;
    }
    uint32_t m = 0;
#pragma unroll
    for (int x = 0; x < 32; ++x) m |= (c0 + x < own && v[x] > thr) ? (1u << x) : 0u;
    while (__any_sync(0xffffffffu, m != 0)) {
      if (m) {
        const int x = __ffs(m) - 1;
        m &= m - 1;
        const float s = pick32(v, x);
        if (s > thr) {
          sift_root(H, K, make_key(s, (int)(c0 + x)));
          thr = key_score(H[0]);
        }
      }
    }
  }
  if (!valid) return;

  const float s_own = St[(own >> 2) * (4 * kRowsS) + tid * 4 + (own & 3)];
  // heap sort: the worst entry moves to the end each round, leaving H best-first
  for (int n = K - 1; n > 0; --n) {
    const uint64_t last = H[n * kThrS];
    H[n * kThrS] = H[0];
    sift_root(H, n, last);
  }
  const float m = K > 0 ? fmaxf(s_own, key_score(H[0])) : s_own;
  float z = 0.f;
  for (int p = K - 1; p >= 0; --p) {
    const uint64_t key = H[p * kThrS];
    if (key) z += __expf(key_score(key) - m);
  }
  z += __expf(s_own - m);
  const float iz = 1.f / z;
  const int64_t r = ((int64_t)b * P.L + i) * P.Hq + h;
  int32_t* ix = idx + r * P.k;
  float* wr = w + r * P.k;
  ix[0] = (int32_t)own;
  wr[0] = __expf(s_own - m) * iz;
  for (int p = 0; p < K; ++p) {
    const uint64_t key = H[p * kThrS];
    ix[p + 1] = key ? key_index(key) : -1;
    wr[p + 1] = key ? __expf(key_score(key) - m) * iz : 0.f;
  }
}

template <int D, int RP>
cudaError_t run_calib(const Params& P, uint8_t* qimg, int T, int64_t n_tiles, int n_sm,
                      cudaStream_t s) {
  constexpr int NR = RP <= 32 ? 2 : 1;
  const size_t sm = sizeof(float) * 2 * D * RP;
  cudaError_t e = set_smem(calib_kernel<D, RP, NR>, sm);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, calib_kernel<D, RP, NR>, kThrS, sm);
  if (e != cudaSuccess) return e;
  const int64_t grid = min((n_tiles + NR - 1) / NR, (int64_t)n_sm * max(1, per_sm));
  HILS_PROFILE("prefill.calib", s);
  calib_kernel<D, RP, NR><<<(unsigned)grid, kThrS, sm, s>>>(P, qimg, T, n_tiles);
  return cudaGetLastError();
}

template <int D>
cudaError_t run_select_tc(const Params& P, const PrefillWs& ws, int32_t* idx, float* w,
                          cudaStream_t s) {
  using Lay = ScoreLayout<D>;
  int dev = 0, n_sm = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return e;
  const int T = (int)((P.L + kRowsS - 1) / kRowsS);
  const int64_t n_tiles = (int64_t)P.B * P.Hq * T;
  uint8_t* qimg = reinterpret_cast<uint8_t*>(ws.qimg);

  const int rp = P.r <= 8 ? 8 : P.r <= 16 ? 16 : P.r <= 32 ? 32 : 64;
  switch (rp) {
    case 8: e = run_calib<D, 8>(P, qimg, T, n_tiles, n_sm, s); break;
    case 16: e = run_calib<D, 16>(P, qimg, T, n_tiles, n_sm, s); break;
    case 32: e = run_calib<D, 32>(P, qimg, T, n_tiles, n_sm, s); break;
    default: e = run_calib<D, 64>(P, qimg, T, n_tiles, n_sm, s); break;
  }
  if (e != cudaSuccess) return e;

  e = set_smem(score_tc_kernel<D>, Lay::kSmem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, score_tc_kernel<D>, kThrS,
                                                    Lay::kSmem);
  if (e != cudaSuccess) return e;
  {
    const int64_t grid = min(n_tiles, (int64_t)n_sm * max(1, per_sm));
    HILS_PROFILE("prefill.score_tc", s);
    score_tc_kernel<D><<<(unsigned)grid, kThrS, Lay::kSmem, s>>>(P, qimg, ws.scores, T, n_tiles,
                                                                 ws.score_cols);
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;

  const size_t hs = sizeof(uint64_t) * kThrS * (size_t)max(1, P.k - 1);
  {
    HILS_PROFILE("prefill.select", s);
    select_kernel<<<(unsigned)n_tiles, kThrS, hs, s>>>(P, ws.scores, T, ws.score_cols, idx, w);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_select_tc(const Params& P, const PrefillWs& ws, int32_t* idx, float* w,
                             cudaStream_t s) {
  return P.d == 64 ? run_select_tc<64>(P, ws, idx, w, s) : run_select_tc<128>(P, ws, idx, w, s);
}

}  // namespace hils
