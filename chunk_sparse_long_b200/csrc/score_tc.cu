// Prefill calibration, landmark scoring, selection and fusion weights (a1-a4)
// for bf16 inputs, as two kernels:
//
//   calib_kernel (a1)   computes q~ = q + (qA)B in float32 per 128-row tile
//       (t = qA first, then t B by column chunks) and splits it into three
//       bf16 terms hi + mid + lo (each the bf16 rounding of what is left, so
//       q~ - (hi + mid + lo) is below 2^-27 |q~|).  The terms are written as
//       ready-made shared-memory images: per 128-row tile, three K-major
//       128-byte-swizzled tiles.
//   score_select_kernel (a2-a4)  persistent and warp-specialised; per
//       128-row tile one bulk copy brings the three term tiles in, and for
//       every block of 128 causally visible chunks S = sum over terms
//       Q_term LM^T runs as 3 x d/16 tcgen05.mma (M = N = 128, float32
//       accumulate) into one of three TMEM buffers while eight epilogue
//       warps read the others back.  The scores never leave the SM: TMEM
//       lane r is query row r of the tile, and two passes over a tile's
//       blocks first bound each row's (k-1)-th best score from below by
//       class maxima, then collect the few candidates above the bound.  A
//       sorting network in registers turns them into the selection, best
//       first, and the softmax of the own and selected scores gives the
//       weights.  Its comment below has the details.
#include <cfloat>

#include "hils_common.cuh"
#include "tc_common.cuh"

namespace hils {
namespace {

constexpr int kRowsS = kScoreTileRows;  // query rows per tile (M)
constexpr int kBlk = kScoreBlock;       // landmark chunks per block (N)
constexpr int kThrS = 128;
constexpr int kTerms = 3;
constexpr int kEpiWarps = 8;          // epilogue warps; warp 8 issues the MMAs and loads
constexpr int kSBufs = 3;             // S buffers of 128 TMEM columns
constexpr uint32_t kTmemColsS = 512;  // the S buffers (allocations are powers of two)
constexpr int kLmBufs = 2;            // landmark blocks in flight: prefetch distance 1
constexpr int kHalfCap = 32;          // selection pass 1: collected candidates per row and column half

template <int D>
struct ScoreLayout {
  static constexpr uint32_t kQt = kRowsS * D * 2;             // one q~ term tile
  static constexpr uint32_t kQimg = kTerms * kQt;             // one tile's three terms
  static constexpr uint32_t kLmB = kBlk * D * 2;              // one landmark block
  static constexpr uint32_t kQ = 0;
  static constexpr uint32_t kLm = kQimg;                      // kLmBufs blocks
  static constexpr uint32_t kBuf = kLm + kLmBufs * kLmB;    // [2][kHalfCap][kThrS] uint64 keys
  static constexpr uint32_t kSmem = kBuf + 2 * kHalfCap * kThrS * 8 + 1024;   // + base alignment
};

// ---- a1: calibration ------------------------------------------------------
// RP = calibration rank rounded up (A staged as [D][RP] with zero columns, B as
// [RP][D] with zero rows).  One CTA of 128 threads takes 128-row tiles in
// turn, in two phases per tile:
//   1. t = q A, float32: thread x computes, for rows x % 64 and x % 64 + 64,
//      the half x / 64 of the RP columns (each 16-byte broadcast load of A
//      feeds 8 FMAs), into shared memory.
//   2. q~ = q + t B, and its split into three bf16 terms: thread (warp w,
//      lane l) owns the 16-byte column chunk c = l % CPR of RPT rows, so one
//      load of a B chunk feeds all of them, and the lanes of a warp store
//      whole 128-byte rows of the swizzled images.
template <int D, int RP>
__global__ void __launch_bounds__(kThrS) calib_kernel(Params P, uint8_t* qimg, int T,
                                                      int64_t n_tiles) {
  using Lay = ScoreLayout<D>;
  constexpr int CPR = D / 8;          // 16-byte chunks per row: 8 or 16
  constexpr int RG = kThrS / CPR;     // row groups in phase 2: 16 or 8
  constexpr int RPT = kRowsS / RG;    // rows per thread in phase 2: 8 or 16
  constexpr int HA = RP / 2;          // rank columns per thread in phase 1
  constexpr int TS = RP + 4;          // padded row of t in shared memory
  extern __shared__ float smf[];
  float* sA = smf;                    // [D][RP]
  float* sB = sA + D * RP;            // [RP][D]
  float* sT = sB + RP * D;            // [kRowsS][TS]
  const int tid = threadIdx.x;
  for (int x = tid; x < D * RP; x += kThrS) {
    const int e = x / RP, a = x % RP;
    sA[x] = a < P.r ? P.A[e * P.r + a] : 0.f;
  }
  for (int x = tid; x < RP * D; x += kThrS) sB[x] = x < P.r * D ? P.Bm[x] : 0.f;
  __syncthreads();
  const uint16_t* qb = reinterpret_cast<const uint16_t*>(P.q);
  auto unpack = [](uint4 u, float (&f)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      f[2 * a] = __uint_as_float(w[a] << 16);
      f[2 * a + 1] = __uint_as_float(w[a] & 0xFFFF0000u);
    }
  };

  for (int64_t gt = blockIdx.x; gt < n_tiles; gt += gridDim.x) {
    const int t = (int)(gt % T);
    const int64_t bh = gt / T;
    const int h = (int)(bh % P.Hq), b = (int)(bh / P.Hq);
    auto row_off = [&](int r, bool& valid) -> int64_t {
      const int64_t i = (int64_t)t * kRowsS + r;
      valid = i < P.L;
      return valid ? (((int64_t)b * P.L + i) * P.Hq + h) * D : 0;
    };
    // ---- phase 1: t = q A (rows r0 and r0 + 64, rank columns a0 .. a0 + HA)
    if (P.r > 0) {
      const int r0 = tid & 63, a0 = (tid >> 6) * HA;
      bool v0, v1;
      const int64_t o0 = row_off(r0, v0), o1 = row_off(r0 + 64, v1);
      float ta[2][HA];
#pragma unroll
      for (int a = 0; a < HA; ++a) ta[0][a] = ta[1][a] = 0.f;
      auto ldq = [&](bool v, int64_t o, int e) -> uint4 {
        return v ? __ldg(reinterpret_cast<const uint4*>(qb + o + e)) : make_uint4(0, 0, 0, 0);
      };
      uint4 q0 = ldq(v0, o0, 0), q1 = ldq(v1, o1, 0);
#pragma unroll 1
      for (int e0 = 0; e0 < D; e0 += 8) {
        // the next 16 bytes are requested before these are used
        const uint4 n0 = e0 + 8 < D ? ldq(v0, o0, e0 + 8) : q0;
        const uint4 n1 = e0 + 8 < D ? ldq(v1, o1, e0 + 8) : q1;
        float f0[8], f1[8];
        unpack(q0, f0);
        unpack(q1, f1);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
#pragma unroll
          for (int a = 0; a < HA; a += 4) {
            const float4 av = *reinterpret_cast<const float4*>(sA + (e0 + u) * RP + a0 + a);
            ta[0][a] = fmaf(f0[u], av.x, ta[0][a]);
            ta[0][a + 1] = fmaf(f0[u], av.y, ta[0][a + 1]);
            ta[0][a + 2] = fmaf(f0[u], av.z, ta[0][a + 2]);
            ta[0][a + 3] = fmaf(f0[u], av.w, ta[0][a + 3]);
            ta[1][a] = fmaf(f1[u], av.x, ta[1][a]);
            ta[1][a + 1] = fmaf(f1[u], av.y, ta[1][a + 1]);
            ta[1][a + 2] = fmaf(f1[u], av.z, ta[1][a + 2]);
            ta[1][a + 3] = fmaf(f1[u], av.w, ta[1][a + 3]);
          }
        }
        q0 = n0;
        q1 = n1;
      }
#pragma unroll
      for (int a = 0; a < HA; a += 4) {
        *reinterpret_cast<float4*>(sT + r0 * TS + a0 + a) =
            make_float4(ta[0][a], ta[0][a + 1], ta[0][a + 2], ta[0][a + 3]);
        *reinterpret_cast<float4*>(sT + (r0 + 64) * TS + a0 + a) =
            make_float4(ta[1][a], ta[1][a + 1], ta[1][a + 2], ta[1][a + 3]);
      }
    }
    __syncthreads();
    // ---- phase 2: q~ = q + t B for chunk c of rows rg, rg + RG, .. (8 at a time)
    const int c = tid % CPR, rg = tid / CPR;
#pragma unroll 1
    for (int j0 = 0; j0 < RPT; j0 += 8) {
      float acc[8][8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        bool v;
        const int64_t o = row_off(rg + RG * (j0 + j), v);
        const uint4 u = v ? __ldg(reinterpret_cast<const uint4*>(qb + o + c * 8))
                          : make_uint4(0, 0, 0, 0);
        unpack(u, acc[j]);
      }
#pragma unroll 1
      for (int a = 0; a < P.r; a += 4) {
        float bv[4][8];
#pragma unroll
        for (int aa = 0; aa < 4; ++aa) {
          const float4 b0 = *reinterpret_cast<const float4*>(sB + (a + aa) * D + c * 8);
          const float4 b1 = *reinterpret_cast<const float4*>(sB + (a + aa) * D + c * 8 + 4);
          bv[aa][0] = b0.x; bv[aa][1] = b0.y; bv[aa][2] = b0.z; bv[aa][3] = b0.w;
          bv[aa][4] = b1.x; bv[aa][5] = b1.y; bv[aa][6] = b1.z; bv[aa][7] = b1.w;
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float4 tv = *reinterpret_cast<const float4*>(sT + (rg + RG * (j0 + j)) * TS + a);
          const float tt[4] = {tv.x, tv.y, tv.z, tv.w};
#pragma unroll
          for (int aa = 0; aa < 4; ++aa)
#pragma unroll
            for (int u = 0; u < 8; ++u) acc[j][u] = fmaf(tt[aa], bv[aa][u], acc[j][u]);
        }
      }
      uint8_t* img = qimg + gt * (int64_t)Lay::kQimg + (uint32_t)(c >> 3) * (kRowsS * 128);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        uint32_t hw[4], mw[4], lw[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          float x0 = acc[j][2 * u], x1 = acc[j][2 * u + 1];
          hw[u] = tc::pack_bf16x2(x0, x1);
          x0 -= __uint_as_float(hw[u] << 16);
          x1 -= __uint_as_float(hw[u] & 0xFFFF0000u);
          mw[u] = tc::pack_bf16x2(x0, x1);
          x0 -= __uint_as_float(mw[u] << 16);
          x1 -= __uint_as_float(mw[u] & 0xFFFF0000u);
          lw[u] = tc::pack_bf16x2(x0, x1);
        }
        const uint32_t off = tc::swz(rg + RG * (j0 + j), c & 7);
        *reinterpret_cast<uint4*>(img + 0 * Lay::kQt + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
        *reinterpret_cast<uint4*>(img + 1 * Lay::kQt + off) = make_uint4(mw[0], mw[1], mw[2], mw[3]);
        *reinterpret_cast<uint4*>(img + 2 * Lay::kQt + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
      }
    }
    __syncthreads();   // t of the next tile goes where this one's was
  }
}

// ---- a1 on the tensor cores ------------------------------------------------
// calib_tc_kernel writes the same q~ images as calib_kernel (rank r <= 32),
// with both small products on the tensor cores.  Per 128-row tile:
//   1. TMA brings the q tile in (K-major, 128-byte swizzle), a tile ahead.
//   2. T = q A.  A is split once per CTA into three bf16 terms (A = A0 + A1
//      + A2 up to 2^-27 |A|); q is bf16, so every product q A_i is exact and
//      T = sum_i q A_i accumulates in float32 in TMEM.
//   3. The epilogue splits T into three bf16 terms T_i and stores them back
//      into TMEM, where the next product reads them as its A operand.
//   4. U = T B = sum over i + j <= 2 of T_i B_j (B split like A; the products
//      left out are below 2^-23 of the largest), float32 in TMEM.
//   5. The epilogue adds q (from the staged tile) to U, splits q~ = q + U
//      into its three bf16 terms and writes them into the tile's three images
//      in shared memory, which one bulk copy stores.
// Warps 0-3: epilogue (TMEM lane quarter w, one query row per thread); warp
// 4: TMA and MMA issue (one thread).
constexpr int kCalibRank = 32;   // rank the tensor-core calibration is built for (r <= 32)
constexpr int kCalibThreads = 160;

template <int D>
struct CalibLayout {
  static constexpr uint32_t kQB = kRowsS * D * 2;        // one q tile = one term image
  static constexpr uint32_t kOpB = kCalibRank * D * 2;   // one term of A (or B) as an operand
  static constexpr uint32_t kQ = 0;                      // two q buffers
  static constexpr uint32_t kA = 2 * kQB;                // A terms: [32 rank rows][D], K-major
  static constexpr uint32_t kB = kA + 3 * kOpB;          // B terms: [32 rank rows][D], MN-major
  static constexpr uint32_t kOut = kB + 3 * kOpB;        // the tile's three q~ term images
  static constexpr uint32_t kSmem = kOut + 3 * kQB + 1024;   // + base alignment
  static_assert(kSmem + 1024 <= 232448, "shared memory above 227 KB");
  // TMEM columns: T (32), its three bf16 terms (16 each), U (D)
  static constexpr uint32_t kT = 0, kTt = 32, kU = 128, kCols = 256;
};

// (x0, x1) -> three packed bf16 pairs, each the rounding of what is left.
__device__ __forceinline__ void split3(float x0, float x1, uint32_t& h, uint32_t& m, uint32_t& l) {
  h = tc::pack_bf16x2(x0, x1);
  x0 -= __uint_as_float(h << 16);
  x1 -= __uint_as_float(h & 0xFFFF0000u);
  m = tc::pack_bf16x2(x0, x1);
  x0 -= __uint_as_float(m << 16);
  x1 -= __uint_as_float(m & 0xFFFF0000u);
  l = tc::pack_bf16x2(x0, x1);
}

template <int D>
__global__ void __launch_bounds__(kCalibThreads, 1) calib_tc_kernel(
    Params P, const __grid_constant__ CUtensorMap tm_q, uint8_t* qimg, int T, int n_tiles) {
  using Lay = CalibLayout<D>;
  constexpr int KB = D / 64;   // 128-byte blocks in a row of D bf16
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t q_full[2], t_full, tt_ready, u_full, out_ready, out_free, drain;
  __shared__ uint32_t tmem_sh;
  __shared__ int abort_sh;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~(uintptr_t)1023);
  const uint32_t sbase = tc::smem_u32(smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // A and B as three bf16 terms each, zero beyond the rank
  for (int x = tid; x < kCalibRank * (D / 8); x += kCalibThreads) {
    const int a = x / (D / 8), c = x % (D / 8);   // rank row, 16-byte chunk along D
    float va[8], vb[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int e = c * 8 + u;
      va[u] = a < P.r ? P.A[e * P.r + a] : 0.f;
      vb[u] = a < P.r ? P.Bm[a * D + e] : 0.f;
    }
    uint32_t ha[4], ma[4], la[4], hb[4], mb[4], lb[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      split3(va[2 * q], va[2 * q + 1], ha[q], ma[q], la[q]);
      split3(vb[2 * q], vb[2 * q + 1], hb[q], mb[q], lb[q]);
    }
    const uint32_t off = (uint32_t)(c >> 3) * (kCalibRank * 128) + tc::swz(a, c & 7);
    *reinterpret_cast<uint4*>(smem + Lay::kA + 0 * Lay::kOpB + off) = make_uint4(ha[0], ha[1], ha[2], ha[3]);
    *reinterpret_cast<uint4*>(smem + Lay::kA + 1 * Lay::kOpB + off) = make_uint4(ma[0], ma[1], ma[2], ma[3]);
    *reinterpret_cast<uint4*>(smem + Lay::kA + 2 * Lay::kOpB + off) = make_uint4(la[0], la[1], la[2], la[3]);
    *reinterpret_cast<uint4*>(smem + Lay::kB + 0 * Lay::kOpB + off) = make_uint4(hb[0], hb[1], hb[2], hb[3]);
    *reinterpret_cast<uint4*>(smem + Lay::kB + 1 * Lay::kOpB + off) = make_uint4(mb[0], mb[1], mb[2], mb[3]);
    *reinterpret_cast<uint4*>(smem + Lay::kB + 2 * Lay::kOpB + off) = make_uint4(lb[0], lb[1], lb[2], lb[3]);
  }
  tc::fence_proxy_async();   // the terms are read by the tensor cores
  if (tid == 0) {
    tc::mbar_init(&q_full[0], 1);
    tc::mbar_init(&q_full[1], 1);
    tc::mbar_init(&t_full, 1);
    tc::mbar_init(&tt_ready, 4);
    tc::mbar_init(&u_full, 1);
    tc::mbar_init(&out_ready, 4);
    tc::mbar_init(&out_free, 1);
    tc::mbar_init(&drain, 1);
    tc::fence_mbar_init();
    abort_sh = 0;
  }
  if (warp == 4) {
    tc::tmem_alloc(&tmem_sh, Lay::kCols);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = tmem_sh;
  volatile int* abort_v = &abort_sh;
  // this CTA's tiles: blockIdx.x, + gridDim.x, ...
  const int my_tiles = ((int)blockIdx.x < n_tiles)
                           ? (n_tiles - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x
                           : 0;
  auto tile_of = [&](int n) { return (int)blockIdx.x + n * (int)gridDim.x; };

  if (warp == 4) {
    if (lane == 0 && my_tiles > 0) {
      constexpr uint32_t kId1 = tc::idesc_bf16(kRowsS, kCalibRank, 0);
      constexpr uint32_t kId2 = tc::idesc_bf16(kRowsS, D, 1);
      auto load_q = [&](int n) {
        const int gt = tile_of(n), t = gt % T, bh = gt / T;
        const int h = bh % P.Hq, b = bh / P.Hq;
        uint64_t* bar = &q_full[n & 1];
        tc::mbar_arrive_expect_tx(bar, Lay::kQB);
#pragma unroll
        for (int c = 0; c < KB; ++c)
          tc::tma_load_4d(sbase + Lay::kQ + (n & 1) * Lay::kQB + c * (kRowsS * 128), &tm_q,
                          c * 64, h, t * kRowsS, b, bar);
      };
      auto mma1 = [&](int n) {   // T = sum_i q A_i
        const uint32_t qb = sbase + Lay::kQ + (n & 1) * Lay::kQB;
#pragma unroll
        for (int term = 0; term < 3; ++term) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t a = tc::smem_desc(qb + (kk >> 2) * (kRowsS * 128) + (kk & 3) * 32, 16, 1024);
            const uint64_t bd = tc::smem_desc(
                sbase + Lay::kA + term * Lay::kOpB + (kk >> 2) * (kCalibRank * 128) + (kk & 3) * 32,
                16, 1024);
            tc::mma_bf16(tmem + Lay::kT, a, bd, kId1, (term | kk) != 0);
          }
        }
        tc::mma_commit(&t_full);
      };
      auto mma2 = [&]() {   // U = sum over i + j <= 2 of T_i B_j
        uint32_t acc = 0;
#pragma unroll
        for (int i = 0; i < 3; ++i) {
#pragma unroll
          for (int j = 0; j + i < 3; ++j) {
#pragma unroll
            for (int kk = 0; kk < kCalibRank / 16; ++kk) {
              const uint64_t bd = tc::smem_desc(sbase + Lay::kB + j * Lay::kOpB + kk * 2048,
                                                kCalibRank * 128, 1024);
              tc::mma_bf16_tmem_a(tmem + Lay::kU, tmem + Lay::kTt + i * 16 + kk * 8, bd, kId2, acc);
              acc = 1;
            }
          }
        }
        tc::mma_commit(&u_full);
      };
      int loads = 0, landed = 0;   // q loads issued / waited for
      bool ok = true, any_mma = false;
      load_q(0);
      loads = 1;
      if (my_tiles > 1) {
        load_q(1);
        loads = 2;
      }
      if (tc::mbar_wait_sleep(&q_full[0], 0, wait_limit())) {
        landed = 1;
        tc::tc_fence_after();
        mma1(0);
        any_mma = true;
      } else {
        ok = false;
      }
      for (int n = 0; ok && n < my_tiles; ++n) {
        // T's terms are in TMEM (and T itself was read): U of tile n
        if (!tc::mbar_wait_sleep(&tt_ready, n & 1, wait_limit()) || *abort_v) {
          ok = false;
          break;
        }
        tc::tc_fence_after();
        mma2();
        if (n + 1 < my_tiles) {
          if (!tc::mbar_wait_sleep(&q_full[(n + 1) & 1], ((n + 1) >> 1) & 1, wait_limit())) {
            ok = false;
            break;
          }
          landed = n + 2;
          tc::tc_fence_after();
          mma1(n + 1);
        }
        // the epilogue has written tile n's images (and read its q tile)
        if (!tc::mbar_wait_sleep(&out_ready, n & 1, wait_limit())) {
          ok = false;
          break;
        }
        tc::bulk_s2g(qimg + (int64_t)tile_of(n) * (3 * Lay::kQB), sbase + Lay::kOut, 3 * Lay::kQB);
        tc::bulk_commit();
        if (n + 2 < my_tiles) {
          load_q(n + 2);
          loads = n + 3;
        }
        tc::bulk_wait_read();
        tc::mbar_arrive(&out_free);
      }
      if (!ok) {
        *abort_v = 1;
        // let what was issued land before the CTA exits (bounded waits)
        for (int x = landed; x < loads; ++x)
          tc::mbar_wait_sleep(&q_full[x & 1], (x >> 1) & 1, kDrainLimitNs);
        if (any_mma) {
          tc::mma_commit(&drain);
          tc::mbar_wait_sleep(&drain, 0, kDrainLimitNs);
        }
      }
      tc::bulk_wait_all();
    }
    __syncwarp();
  } else {
    // ---- epilogue: warp w owns TMEM lanes 32 w .. 32 w + 31 (tile rows) ----
    const int row = warp * 32 + lane;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    bool ok = true;
    for (int n = 0; n < my_tiles; ++n) {
      // T -> three bf16 terms, back into TMEM as the next product's A operand
      if (!tc::warp_wait(&t_full, n & 1, wait_limit()) || *abort_v) {
        ok = false;
        break;
      }
      tc::tc_fence_after();
      {
        uint32_t tv[32];
        tc::tmem_ld32(tmem + lane_off + Lay::kT, tv);
        tc::tmem_ld_wait();
        uint32_t th[16], tm[16], tl[16];
#pragma unroll
        for (int x = 0; x < 16; ++x)
          split3(__uint_as_float(tv[2 * x]), __uint_as_float(tv[2 * x + 1]), th[x], tm[x], tl[x]);
        tc::tmem_st16(tmem + lane_off + Lay::kTt, th);
        tc::tmem_st16(tmem + lane_off + Lay::kTt + 16, tm);
        tc::tmem_st16(tmem + lane_off + Lay::kTt + 32, tl);
        tc::tmem_st_wait();
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&tt_ready);
      // q~ = q + U, split into three terms, into the output images
      if (!tc::warp_wait(&u_full, n & 1, wait_limit()) ||
          (n > 0 && !tc::warp_wait(&out_free, (n - 1) & 1, wait_limit()))) {
        ok = false;
        break;
      }
      tc::tc_fence_after();
      const uint8_t* qt = smem + Lay::kQ + (n & 1) * Lay::kQB;
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t uv[32];
        tc::tmem_ld32(tmem + lane_off + Lay::kU + c0, uv);
        tc::tmem_ld_wait();
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          const int c = c0 / 8 + cc;   // 16-byte chunk of the row
          const uint32_t off = (uint32_t)(c >> 3) * (kRowsS * 128) + tc::swz(row, c & 7);
          const uint4 qv = *reinterpret_cast<const uint4*>(qt + off);
          const uint32_t qw[4] = {qv.x, qv.y, qv.z, qv.w};
          uint32_t h[4], m[4], l[4];
#pragma unroll
          for (int q = 0; q < 4; ++q)
            split3(__uint_as_float(qw[q] << 16) + __uint_as_float(uv[cc * 8 + 2 * q]),
                   __uint_as_float(qw[q] & 0xFFFF0000u) + __uint_as_float(uv[cc * 8 + 2 * q + 1]),
                   h[q], m[q], l[q]);
          *reinterpret_cast<uint4*>(smem + Lay::kOut + 0 * Lay::kQB + off) = make_uint4(h[0], h[1], h[2], h[3]);
          *reinterpret_cast<uint4*>(smem + Lay::kOut + 1 * Lay::kQB + off) = make_uint4(m[0], m[1], m[2], m[3]);
          *reinterpret_cast<uint4*>(smem + Lay::kOut + 2 * Lay::kQB + off) = make_uint4(l[0], l[1], l[2], l[3]);
        }
      }
      tc::tc_fence_before();
      tc::fence_proxy_async();   // the images are read by the bulk copy
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&out_ready);
    }
    if (!ok) *abort_v = 1;
  }
  if (tid == 0 && *abort_v) set_device_error(kErrTimeout);
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 4) tc::tmem_dealloc(tmem, Lay::kCols);
}

template <int D>
cudaError_t run_calib_tc(const Params& P, uint8_t* qimg, int T, int64_t n_tiles, int n_sm,
                         cudaStream_t s) {
  using Lay = CalibLayout<D>;
  CUtensorMap tm;
  {
    // q [B][L][Hq][D] as (D, head, position, sequence); a box is 64 elements of
    // 128 consecutive positions of one head
    const uint64_t dims[4] = {(uint64_t)D, (uint64_t)P.Hq, (uint64_t)P.L, (uint64_t)P.B};
    const uint64_t strides[3] = {(uint64_t)D * 2, (uint64_t)P.Hq * D * 2,
                                 (uint64_t)P.L * P.Hq * D * 2};
    const uint32_t box[4] = {64, 1, (uint32_t)kRowsS, 1};
    cudaError_t e = encode_tmap_bf16(&tm, 4, P.q, dims, strides, box);
    if (e != cudaSuccess) return e;
  }
  cudaError_t e = set_smem(calib_tc_kernel<D>, Lay::kSmem);
  if (e != cudaSuccess) return e;
  const int64_t grid = min(n_tiles, (int64_t)n_sm);
  HILS_PROFILE("prefill.calib", s);
  calib_tc_kernel<D><<<(unsigned)grid, kCalibThreads, Lay::kSmem, s>>>(P, tm, qimg, T, (int)n_tiles);
  return cudaGetLastError();
}

// ---- a2-a4: landmark scores, selection and weights, fused -------------------
// Keys: a larger key ranks higher in (score desc, index asc).  The high word
// is the score's bits mapped to an unsigned order (-0 taken as +0), the low
// word is ~j.  Key 0 is an empty slot, below every real entry.
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

// Sifts x down from slot p of the min-heap H[0 .. size) (stride kThrS).
__device__ __forceinline__ void sift_down(uint64_t* H, int size, int p, uint64_t x) {
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

// Keeps the best K of the n >= K keys in H[0 .. n) as a min-heap in
// H[0 .. K): its root is then the K-th best.
__device__ __forceinline__ void keep_best(uint64_t* H, int n, int K) {
  for (int p = K / 2 - 1; p >= 0; --p) sift_down(H, K, p, H[p * kThrS]);
  for (int e = K; e < n; ++e) {
    const uint64_t x = H[e * kThrS];
    if (x > H[0]) sift_down(H, K, 0, x);
  }
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

// Bitonic sorting network over N registers, descending.
template <int N, typename T>
__device__ __forceinline__ void sort_desc(T (&a)[N]) {
#pragma unroll
  for (int k = 2; k <= N; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
#pragma unroll
      for (int i = 0; i < N; ++i) {
        const int l = i ^ j;
        if (l > i) {
          const T x = a[i], y = a[l];
          const bool sw = ((i & k) == 0) ? (x < y) : (y < x);
          a[i] = sw ? y : x;
          a[l] = sw ? x : y;
        }
      }
    }
  }
}

// Sorts a bitonic sequence of N registers descending (half-cleaner cascade).
template <int N, typename T>
__device__ __forceinline__ void merge_desc(T (&a)[N]) {
#pragma unroll
  for (int j = N >> 1; j > 0; j >>= 1) {
#pragma unroll
    for (int i = 0; i < N; ++i) {
      if ((i & j) == 0) {
        const T x = a[i], y = a[i + j];
        const bool sw = x < y;
        a[i] = sw ? y : x;
        a[i + j] = sw ? x : y;
      }
    }
  }
}

// One (tile, pass, landmark block) step of a CTA's walk.  Walk position w
// covers (sequence, head) w / T and tile T - 1 - w % T: the tiles with the
// most blocks come first, so the walk ends on short tiles.  Every tile takes
// two passes over its blocks.
struct Step {
  int w;    // walk position; >= n_tiles once the walk is over
  int bh;   // b * Hq + h
  int t, pass, blk, nblk;
};

__device__ __forceinline__ void step_set(Step& s, int w, const Params& P, int T, int n_tiles) {
  s.w = w;
  s.pass = 0;
  s.blk = 0;
  if (w < n_tiles) {
    s.bh = (int)((unsigned)w / (unsigned)T);
    s.t = T - 1 - (w - s.bh * T);
    s.nblk = (int)score_tile_blocks(P.L, P.pos0, s.t);
  } else {
    s.bh = 0;
    s.t = 0;
    s.nblk = 0;
  }
}

__device__ __forceinline__ void step_next(Step& s, const Params& P, int T, int n_tiles) {
  if (++s.blk < s.nblk) return;
  if (s.pass == 0) {
    s.pass = 1;
    s.blk = 0;
  } else {
    step_set(s, s.w + (int)gridDim.x, P, T, n_tiles);
  }
}

// Persistent: each CTA walks its tiles.  Warp 8 issues: per tile one bulk
// copy brings the q~ term images in, and per landmark block of 128 chunks (a
// TMA load from the [B][max_chunks][Hkv][d] landmark tensor, already in the
// swizzled K-major layout) the MMAs accumulate S into one of three TMEM
// buffers.  Warps 0-7 read them back: warps q and q + 4 share TMEM lanes
// 32q .. 32q+31, the tile's rows, and take the first and the second 64
// columns of every block.
//
// Selection in two passes over the tile's blocks, so that no per-score work
// depends on earlier scores:
//   pass 0  per row and column half, the maximum score of each column class
//           of candidates j < own, kept in registers between blocks: over
//           both halves, the maxima of the 128 classes j mod 128.  The K-th
//           largest of these maxima (K = k-1) is a lower bound tau on the
//           row's K-th best score: the K classes it comes from hold K
//           distinct candidates scoring at least tau.  The two halves swap
//           their best 32 maxima to find it.
//   pass 1  the same scores again; every candidate scoring at least tau is
//           appended to its half's buffer in shared memory (column = row).
//           On random scores that is a few more than K per row.  A half
//           buffer that fills up is cut to its own best K, whose K-th best
//           then becomes an exact bar for that half.
// After pass 1 each half sorts its buffer and the first half merges in the
// second's: the best K are the selection, best first.  A candidate left out
// scores below tau, or below a half's bar, so at least K collected ones rank
// above it.  The softmax of the own and selected scores gives the weights.
// Both passes compare raw accumulator values; pass 1's bound is lowered by a
// few ulps, so every score whose scaled value could round up to the bound's
// is collected, and the keys (scaled scores) then decide exactly.
template <int D>
__global__ void __launch_bounds__(2 * kThrS + 32, 1) score_select_kernel(
    Params P, const __grid_constant__ CUtensorMap tm_lm, const uint8_t* qimg, int T, int n_tiles,
    int32_t* idx, float* wout) {
  using Lay = ScoreLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t s_full[kSBufs];   // MMAs into S buffer b done
  __shared__ uint64_t s_free[kSBufs];   // the eight epilogue warps have read S buffer b
  __shared__ uint64_t lm_bar[kLmBufs];  // landmark buffer b landed
  __shared__ uint64_t qbar;             // q~ terms of the current tile landed
  __shared__ uint32_t tmem_sh;
  __shared__ int abort_sh;
  __shared__ float s_own_sh[kRowsS];  // each row's own-chunk score, from whichever half saw it
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~(uintptr_t)1023);
  const uint32_t sbase = tc::smem_u32(smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if ((int)blockIdx.x >= n_tiles) return;

  if (tid == 0) {
    for (int b = 0; b < kSBufs; ++b) {
      tc::mbar_init(&s_full[b], 1);
      tc::mbar_init(&s_free[b], kEpiWarps);
    }
    for (int b = 0; b < kLmBufs; ++b) tc::mbar_init(&lm_bar[b], 1);
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
  volatile int* abort_v = &abort_sh;

  if (warp == kEpiWarps) {
    // ---- MMA and TMA issue (one thread) ----
    if (lane == 0) {
      constexpr uint32_t kId = tc::idesc_bf16(kRowsS, kBlk, 0);
      auto load_q = [&](const Step& st) {
        const uint8_t* src = qimg + ((int64_t)st.bh * T + st.t) * (int64_t)Lay::kQimg;
        tc::mbar_arrive_expect_tx(&qbar, Lay::kQimg);
#pragma unroll
        for (int term = 0; term < kTerms; ++term)
          tc::bulk_g2s(sbase + Lay::kQ + term * Lay::kQt, src + term * Lay::kQt, Lay::kQt, &qbar);
      };
      auto load_lm = [&](const Step& s, int nb) {
        const int b = (int)((unsigned)s.bh / (unsigned)P.Hq);
        const int g = (int)((unsigned)(s.bh - b * P.Hq) / (unsigned)P.group);
        const uint32_t dst = sbase + Lay::kLm + (uint32_t)nb * Lay::kLmB;
        tc::mbar_arrive_expect_tx(&lm_bar[nb], Lay::kLmB);
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          tc::tma_load_4d(dst + c * (kBlk * 128), &tm_lm, c * 64, g, s.blk * kBlk, b, &lm_bar[nb]);
      };
      // waits for the MMAs of step m
      auto mma_done = [&](int m, uint64_t limit) {
        return tc::mbar_wait_sleep(&s_full[m % kSBufs], (uint32_t)(m / kSBufs) & 1u, limit);
      };
      Step st, pf;
      step_set(st, blockIdx.x, P, T, n_tiles);
      pf = st;
      load_lm(pf, 0);
      step_next(pf, P, T, n_tiles);
      int n = 0;
      int lm_issued = 1;   // landmark loads issued (steps 0 .. lm_issued-1)
      int mma_issued = 0;  // steps whose MMAs were committed
      uint32_t qphase = 0;
      bool q_pending = false;
      bool ok = true;
      for (; st.w < n_tiles; step_next(st, P, T, n_tiles), ++n) {
        if (*abort_v) {
          ok = false;
          break;
        }
        if (st.pass == 0 && st.blk == 0) {
          // the previous tile's MMAs must be done before its q~ terms are replaced
          if (n > 0 && !mma_done(n - 1, wait_limit())) {
            ok = false;
            break;
          }
          load_q(st);
          q_pending = true;
          {
            // the CTA's next tile: its q~ terms into L2 while this tile runs
            Step nx;
            step_set(nx, st.w + (int)gridDim.x, P, T, n_tiles);
            if (nx.w < n_tiles)
              tc::bulk_prefetch_l2(qimg + ((int64_t)nx.bh * T + nx.t) * (int64_t)Lay::kQimg,
                                   Lay::kQimg);
          }
          if (!tc::mbar_wait_sleep(&qbar, qphase, wait_limit())) {
            ok = false;
            break;
          }
          q_pending = false;
          qphase ^= 1;
        }
        const int sb = n % kSBufs;
        if (n >= kSBufs &&
            !tc::mbar_wait_sleep(&s_free[sb], (uint32_t)(n / kSBufs - 1) & 1u, wait_limit())) {
          ok = false;
          break;
        }
        if (!tc::mbar_wait_sleep(&lm_bar[n & 1], (uint32_t)(n >> 1) & 1u, wait_limit())) {
          ok = false;
          break;
        }
        tc::tc_fence_after();
        const uint32_t lm = sbase + Lay::kLm + (uint32_t)(n & 1) * Lay::kLmB;
#pragma unroll
        for (int term = 0; term < kTerms; ++term) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t a = tc::smem_desc(sbase + Lay::kQ + term * Lay::kQt +
                                                 (kk >> 2) * (kRowsS * 128) + (kk & 3) * 32,
                                             16, 1024);
            const uint64_t bd =
                tc::smem_desc(lm + (kk >> 2) * (kBlk * 128) + (kk & 3) * 32, 16, 1024);
            tc::mma_bf16(tmem + sb * kBlk, a, bd, kId, (term | kk) != 0);
          }
        }
        tc::mma_commit(&s_full[sb]);
        mma_issued = n + 1;
        // step n+1's landmark block goes where step n-1's was: its MMAs must be done
        if (pf.w < n_tiles) {
          if (n > 0 && !mma_done(n - 1, wait_limit())) {
            ok = false;
            break;
          }
          load_lm(pf, (n + 1) & 1);
          ++lm_issued;
          step_next(pf, P, T, n_tiles);
        }
      }
      if (!ok) {
        *abort_v = 1;
        // let what was issued land before the CTA exits (bounded waits)
        if (mma_issued > 0) mma_done(mma_issued - 1, kDrainLimitNs);
        for (int m = mma_issued; m < lm_issued; ++m)
          tc::mbar_wait_sleep(&lm_bar[m & 1], (uint32_t)(m >> 1) & 1u, kDrainLimitNs);
        if (q_pending) tc::mbar_wait_sleep(&qbar, qphase, kDrainLimitNs);
      }
    }
  } else {
    // ---- epilogue: eight warps.  Warps q and q + 4 share TMEM lanes 32q ..
    // 32q + 31 (query rows of the tile) and take the first and the second 64
    // columns of every block: two warps per SM sub-partition, so one hides the
    // other's dependent-instruction latency.  Each half keeps its own class
    // maxima (classes j mod 128 over the two halves) and its own collection
    // buffer; the pair meets on a named barrier to combine them.
    const int q = warp & 3, hf = warp >> 2;
    const int row = q * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const int co = hf * 64;
    const int bar_id = 1 + q;
    const int K = P.k - 1;
    uint64_t* const buf = reinterpret_cast<uint64_t*>(smem + Lay::kBuf);
    uint64_t* Bf = buf + hf * kHalfCap * kThrS + row;         // this half, stride kThrS
    uint64_t* Bo = buf + (1 - hf) * kHalfCap * kThrS + row;   // the partner's half
    float thr_f = -INFINITY;   // pass 1: raw scores below this are left out
    uint64_t thr_key = 0;      // pass 1: and keys must exceed this (set once the buffer was cut)
    int cnt = 0;               // pass 1: keys in this half's buffer
    const float sqrt_d = sqrtf((float)P.d);

    auto append = [&](uint64_t key) {
      Bf[cnt * kThrS] = key;
      if (++cnt == kHalfCap) {
        keep_best(Bf, cnt, K);
        cnt = K;
        thr_key = Bf[0];
        // the bar in raw units, lowered by a few ulps: the keys decide exactly
        const float r = key_score(thr_key) * sqrt_d;
        thr_f = fmaxf(thr_f, r - fabsf(r) * 0x1p-20f);
      }
    };

    // Both halves sort their buffers (one sorting network in registers); the
    // second half hands its sorted keys over, and the first merges them in: the
    // slot-wise maximum of its list and the reversed other list holds the best
    // 32 of both as a bitonic sequence, which a half-cleaner cascade sorts.  The
    // top K, best first, and the own chunk's score give idx and w.
    auto finish_tile = [&](const Step& st) {
      uint64_t c[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) c[e] = e < cnt ? Bf[e * kThrS] : 0ull;
      sort_desc<32>(c);
      if (hf == 1) {
#pragma unroll
        for (int e = 0; e < 32; ++e) Bf[e * kThrS] = c[e];
      }
      tc::named_barrier(bar_id, 64);
      if (hf == 0) {
#pragma unroll
        for (int p = 0; p < 32; ++p) {
          const uint64_t y = Bo[(31 - p) * kThrS];
          c[p] = c[p] > y ? c[p] : y;
        }
        merge_desc<32>(c);
        const int i = st.t * kRowsS + row;
        if (i < P.L) {
          const int b = (int)((unsigned)st.bh / (unsigned)P.Hq);
          const int h = st.bh - b * P.Hq;
          const int own = (int)((P.pos0 + i) / kChunk);
          const float s_own = s_own_sh[row];
          const float mx = K > 0 ? fmaxf(s_own, key_score(c[0])) : s_own;
          float sc[kMaxTopK];
          float z = 0.f;
#pragma unroll
          for (int p = 0; p < kMaxTopK; ++p) {
            const float e =
                p == 0 ? __expf(s_own - mx)
                       : ((p - 1 < K && c[p - 1]) ? __expf(key_score(c[p - 1]) - mx) : 0.f);
            sc[p] = e;
            z += e;
          }
          const float iz = 1.f / z;
          const int64_t r = ((int64_t)b * P.L + i) * P.Hq + h;
          int32_t* ix = idx + r * P.k;
          float* wr = wout + r * P.k;
          auto jat = [&](int p) -> int32_t {
            return p == 0 ? own : (c[p - 1] ? key_index(c[p - 1]) : -1);
          };
          // 16-byte stores when every row starts 16-byte aligned (the output
          // pointers are the caller's: only 4-byte alignment is required)
          const bool vec = (P.k & 3) == 0 &&
                           ((reinterpret_cast<uintptr_t>(idx) | reinterpret_cast<uintptr_t>(wout)) &
                            15u) == 0;
          if (vec) {
#pragma unroll
            for (int p = 0; p < kMaxTopK; p += 4) {
              if (p < P.k) {
                *reinterpret_cast<int4*>(ix + p) =
                    make_int4(jat(p), jat(p + 1), jat(p + 2), jat(p + 3));
                *reinterpret_cast<float4*>(wr + p) =
                    make_float4(sc[p] * iz, sc[p + 1] * iz, sc[p + 2] * iz, sc[p + 3] * iz);
              }
            }
          } else {
#pragma unroll
            for (int p = 0; p < kMaxTopK; ++p) {
              if (p < P.k) {
                ix[p] = jat(p);
                wr[p] = sc[p] * iz;
              }
            }
          }
        }
      }
      cnt = 0;
      thr_key = 0;
    };

    // S buffer sb, this half's 64 columns: tile st's rows against chunks
    // st.blk * 128 + co ..
    // Pass 0 keeps this half's 64 class maxima in registers from block to
    // block (raw accumulator values).
    float cmx[64];
    auto drain = [&](int sb, const Step& st) {
      const int i = st.t * kRowsS + row;
      const int i_last = min((st.t + 1) * kRowsS, (int)P.L) - 1;
      const int own = i < P.L ? (int)((P.pos0 + i) / kChunk) : 0;
      const int own_min = (int)((P.pos0 + st.t * kRowsS) / kChunk);
      const int own_max = (int)((P.pos0 + i_last) / kChunk);
      const int jb = st.blk * kBlk + co;
      const uint32_t ta = tmem + sb * kBlk + co + lane_off;
      if (st.pass == 0) {
        if (K == 0) return;
        if (st.blk == 0) {
#pragma unroll
          for (int x = 0; x < 64; ++x) cmx[x] = -INFINITY;
        }
        if (jb < own_max) {
          uint32_t s0[32], s1[32];
          tc::tmem_ld32(ta, s0);
          tc::tmem_ld32(ta + 32, s1);
          tc::tmem_ld_wait();
          if (jb + 64 <= own_min) {
#pragma unroll
            for (int x = 0; x < 32; ++x) {
              cmx[x] = fmaxf(cmx[x], __uint_as_float(s0[x]));
              cmx[32 + x] = fmaxf(cmx[32 + x], __uint_as_float(s1[x]));
            }
          } else {
#pragma unroll
            for (int x = 0; x < 32; ++x) {
              cmx[x] = fmaxf(cmx[x], jb + x < own ? __uint_as_float(s0[x]) : -INFINITY);
              cmx[32 + x] = fmaxf(cmx[32 + x], jb + 32 + x < own ? __uint_as_float(s1[x]) : -INFINITY);
            }
          }
        }
        if (st.blk == st.nblk - 1) {
          float cm[64];
#pragma unroll
          for (int x = 0; x < 64; ++x) cm[x] = cmx[x];
          sort_desc<64>(cm);
          // the two halves' best 32 maxima meet in the (empty) collection
          // buffers: the K-th largest of all 128 class maxima is the bound
          tc::named_barrier(bar_id, 64);   // the partner is done with the last finish
#pragma unroll
          for (int s = 0; s < 32; ++s) Bf[s * kThrS] = __float_as_uint(cm[s]);
          tc::named_barrier(bar_id, 64);
#pragma unroll
          for (int p = 0; p < 32; ++p) cm[p] = fmaxf(cm[p], __uint_as_float((uint32_t)Bo[(31 - p) * kThrS]));
          tc::named_barrier(bar_id, 64);   // read before pass 1 appends
          float top[32];
#pragma unroll
          for (int p = 0; p < 32; ++p) top[p] = cm[p];
          merge_desc<32>(top);
          float tau = top[0];
#pragma unroll
          for (int p = 1; p < 32; ++p) tau = (p == K - 1) ? top[p] : tau;
          // pass 1 compares raw scores with this bound, lowered by a few
          // ulps so that every score whose scaled value could round to the
          // bound's scaled value is collected too
          thr_f = tau - fabsf(tau) * 0x1p-20f;
        }
        return;
      }
      if (jb <= own_max) {
        uint32_t sv[2][32];
        tc::tmem_ld32(ta, sv[0]);
        tc::tmem_ld32(ta + 32, sv[1]);
        tc::tmem_ld_wait();
        float v0[32], v1[32];
#pragma unroll
        for (int x = 0; x < 32; ++x) {
          v0[x] = __uint_as_float(sv[0][x]);
          v1[x] = __uint_as_float(sv[1][x]);
        }
        const int od = own - jb;
        if (od >= 0 && od < 32) s_own_sh[row] = pick32(v0, od) * P.inv_sqrt_d;
        if (od >= 32 && od < 64) s_own_sh[row] = pick32(v1, od - 32) * P.inv_sqrt_d;
        if (K > 0 && jb < own_max) {
          uint32_t m0 = 0, m1 = 0;
          if (jb + 64 <= own_min) {
#pragma unroll
            for (int x = 0; x < 32; ++x) {
              m0 |= v0[x] >= thr_f ? (1u << x) : 0u;
              m1 |= v1[x] >= thr_f ? (1u << x) : 0u;
            }
          } else {
#pragma unroll
            for (int x = 0; x < 32; ++x) {
              m0 |= (jb + x < own && v0[x] >= thr_f) ? (1u << x) : 0u;
              m1 |= (jb + 32 + x < own && v1[x] >= thr_f) ? (1u << x) : 0u;
            }
          }
          // per round one candidate of each 32 columns per lane: lanes do not
          // serialise each other, and the two extractions are independent;
          // keys hold the scaled scores
          while (__any_sync(0xffffffffu, (m0 | m1) != 0)) {
            if (m0) {
              const int x = __ffs(m0) - 1;
              m0 &= m0 - 1;
              const uint64_t key = make_key(pick32(v0, x) * P.inv_sqrt_d, jb + x);
              if (key > thr_key) append(key);
            }
            if (m1) {
              const int x = __ffs(m1) - 1;
              m1 &= m1 - 1;
              const uint64_t key = make_key(pick32(v1, x) * P.inv_sqrt_d, jb + 32 + x);
              if (key > thr_key) append(key);
            }
          }
        }
      }
      if (st.blk == st.nblk - 1) finish_tile(st);
    };

    Step st;
    step_set(st, blockIdx.x, P, T, n_tiles);
    for (int n = 0; st.w < n_tiles; step_next(st, P, T, n_tiles), ++n) {
      const int sb = n % kSBufs;
      const bool got = tc::mbar_wait_sleep(&s_full[sb], (uint32_t)(n / kSBufs) & 1u, wait_limit());
      // the pair decides together, so neither is ever left alone at its named barrier
      if (tc::named_barrier_or(bar_id, 64, !got || *abort_v != 0)) {
        if (lane == 0) *abort_v = 1;
        break;
      }
      tc::tc_fence_after();
      drain(sb, st);
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&s_free[sb]);
    }
  }

  if (tid == 0 && *abort_v) set_device_error(kErrTimeout);
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, kTmemColsS);
}

template <int D, int RP>
cudaError_t run_calib(const Params& P, uint8_t* qimg, int T, int64_t n_tiles, int n_sm,
                      cudaStream_t s) {
  const size_t sm = sizeof(float) * (2 * D * RP + kRowsS * (RP + 4));
  cudaError_t e = set_smem(calib_kernel<D, RP>, sm);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, calib_kernel<D, RP>, kThrS, sm);
  if (e != cudaSuccess) return e;
  const int64_t grid = min(n_tiles, (int64_t)n_sm * max(1, per_sm));
  HILS_PROFILE("prefill.calib", s);
  calib_kernel<D, RP><<<(unsigned)grid, kThrS, sm, s>>>(P, qimg, T, n_tiles);
  return cudaGetLastError();
}

template <int D>
cudaError_t landmark_tmap(const Params& P, CUtensorMap* tm) {
  const uint64_t dims[4] = {(uint64_t)D, (uint64_t)P.Hkv, (uint64_t)P.max_chunks, (uint64_t)P.B};
  const uint64_t strides[3] = {(uint64_t)D * 2, (uint64_t)P.Hkv * D * 2,
                               (uint64_t)P.max_chunks * P.Hkv * D * 2};
  const uint32_t box[4] = {64, 1, (uint32_t)kBlk, 1};
  return encode_tmap_bf16(tm, 4, P.landmarks, dims, strides, box);
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

  // ranks up to 32 on the tensor cores, larger ones (up to 64) on the CUDA cores
  e = P.r <= kCalibRank ? run_calib_tc<D>(P, qimg, T, n_tiles, n_sm, s)
                        : run_calib<D, 64>(P, qimg, T, n_tiles, n_sm, s);
  if (e != cudaSuccess) return e;

  CUtensorMap tm;
  if ((e = landmark_tmap<D>(P, &tm)) != cudaSuccess) return e;
  const size_t smem = Lay::kSmem;
  e = set_smem(score_select_kernel<D>, smem);
  if (e != cudaSuccess) return e;
  const int64_t grid = min(n_tiles, (int64_t)n_sm);
  HILS_PROFILE("prefill.score_select", s);
  score_select_kernel<D><<<(unsigned)grid, 2 * kThrS + 32, smem, s>>>(P, tm, qimg, T, (int)n_tiles, idx, w);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_select_tc(const Params& P, const PrefillWs& ws, int32_t* idx, float* w,
                             cudaStream_t s) {
  return P.d == 64 ? run_select_tc<64>(P, ws, idx, w, s) : run_select_tc<128>(P, ws, idx, w, s);
}

}  // namespace hils
