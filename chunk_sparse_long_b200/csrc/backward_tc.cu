// Prefill backward for bf16 storage at head_dim 128: the attention products
// on the tensor cores, and the score path folded into per-item sums.
//
// Each work item of the key-major buckets (up to 128 pairs of one chunk j and
// KV head) is one tile of M = 128 rows, one per pair.  With Q the pairs'
// query rows, G = w dout their weighted output gradients, and K, V the
// chunk's keys and values:
//   S = Q K^T,  P = softmax(S / sqrt(d)) over the visible keys,  O = P V,
//   dw = dout . O,  dP = G V^T,  dS = P (dP - w dw),
//   dQ = dS K / sqrt(d),  dK^T = Q^T dS / sqrt(d),  dV^T = G^T P.
// These are six tcgen05 products per tile, all with M = 128: dK and dV are
// taken transposed, so that their M is the head dimension.  Operands are bf16
// in shared memory (128-byte swizzle); P, G and dS are rounded to bf16 as the
// tensor cores take them.  Accumulators are float32 in tensor memory:
//   columns [0, 64)   S, then dP
//           [64, 192) O, then dQ
//           [192, 256) dK^T,  [256, 320) dV^T
// One thread per tile row (4 warps; warp w reads TMEM lanes 32w .. 32w + 31)
// does the element-wise work, and thread 0 issues the products.  The kernel
// is persistent: one CTA per SM walks the items.
//
// The score path.  The fusion softmax's row term sum_l w_l dw_l equals
// dout . out, so with the forward's output it is known before the attention
// pass (delta); then ds = w (dw - delta) is known inside the tile.  The
// calibration q~ = q + (qA)B is linear, which folds the rest into per-item
// sums.  With v = sum over the item's pairs of ds q (a d-vector):
//   dq     += ds lm'_j / sqrt(d),  lm'_j = lm_j + (lm_j B^T) A^T  (per chunk,
//             precomputed; added with the tile's dQ)
//   dlm_j  += (v_j + (v_j A) B) / sqrt(d)       (v_j summed over chunk j's pairs)
//   dA     += M B^T / sqrt(d),  dB += A^T M / sqrt(d),  M = sum over chunks of v_j lm_j^T
// so no per-row pass over the k selected landmarks remains.  v is one more
// column of the dK^T product (N = 80, ds as its B column).  A CTA walks a
// contiguous range of items, so dK^T, dV^T and v add up in tensor memory over
// the items of one key and go out once per run.  dq and the
// gradients of the pool and the landmarks receive float32 additions in L2.
// The CUDA-core kernels for the other configurations are in backward.cu.
#include "hils_common.cuh"
#include "tc_common.cuh"

namespace hils {
namespace {

constexpr int kD = 128;
constexpr int kRowsT = 128;                          // tile rows: pairs
constexpr int kThreadsT = 128;
constexpr uint32_t kQB = kRowsT * kD * 2;            // Q or G tile: two 64-column blocks of 16 KB
constexpr uint32_t kKVB = kChunk * kD * 2;           // K or V tile: two blocks of 8 KB
constexpr uint32_t kPB = kRowsT * kChunk * 2;        // P or dS tile: one block of 16 KB
struct TLay {
  static constexpr uint32_t kQ = 0;
  static constexpr uint32_t kG = kQ + kQB;
  static constexpr uint32_t kK = kG + kQB;
  static constexpr uint32_t kV = kK + kKVB;
  static constexpr uint32_t kP = kV + kKVB;
  static constexpr uint32_t kS = kP + kPB;          // dS, then one more block whose
                                                     // column 0 holds ds
  static constexpr uint32_t kStage = kS + 2 * kPB;   // per warp 32 rows x 32 floats of dQ
  static constexpr uint32_t kStageLd = 36;           // floats per staged row (16-byte rows)
  static constexpr uint32_t kBytes = kStage + 4 * 32 * kStageLd * 4;   // 162 KB
};
// TMEM columns: S / dP, O / dQ (per item); dK^T with v in its column 64, and
// dV^T (summed over a run of items of one key)
constexpr uint32_t kColS = 0, kColO = 64, kColDK = 192, kColV = 256, kColDV = 272,
                   kTmemCols = 512;

// Byte offset of 16-byte chunk c of row r in a K-major tile of `rows` rows
// (64-column blocks one after another, 128-byte swizzle inside each).
__device__ __forceinline__ uint32_t tile_at(uint32_t rows, int r, int c) {
  return (uint32_t)(c >> 3) * (rows * 128u) + tc::swz((uint32_t)r, (uint32_t)(c & 7));
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// All threads wait for the products committed last; false (everywhere) if any
// thread's bounded wait ran out.
__device__ __forceinline__ bool wait_products(uint64_t* bar, uint32_t& phase) {
  const bool good = tc::mbar_wait(bar, phase, wait_limit());
  phase ^= 1u;
  return __syncthreads_and(good) != 0;
}

__global__ void __launch_bounds__(kThreadsT, 1)
    attn_bwd_tc_kernel(Params P, PrefillWs ws, const float* wts, const void* dout,
                       const float* delta, const float* lmc, float* vchunk, float* dq,
                       float* dpages) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t mma_bar;
  __shared__ uint32_t tmem_sh;
  __shared__ float slm[kD];        // the item's lm'_j
  __shared__ float sds[kRowsT];    // ds of every tile row (0 past the item's pairs)
  __shared__ int32_t srow[kRowsT]; // query row of every tile row (-1 past the item's pairs)
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~(uintptr_t)1023);
  const uint32_t sb = tc::smem_u32(smem);
  const int tid = threadIdx.x, warp = tid >> 5;
  if (warp == 0) {
    tc::tmem_alloc(&tmem_sh, kTmemCols);
    tc::tmem_relinquish();
  }
  if (tid == 0) {
    tc::mbar_init(&mma_bar, 1);
    tc::fence_mbar_init();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = tmem_sh;
  const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);   // this warp's TMEM lanes
  constexpr uint32_t kIdS = tc::idesc_bf16(kRowsT, kChunk, 0);        // N = 64, B K-major
  constexpr uint32_t kIdO = tc::idesc_bf16(kRowsT, kD, 1);            // N = d, B MN-major
  constexpr uint32_t kIdT = tc::idesc_bf16_ab(kD, kChunk, 1, 1);      // M = d, N = 64, both MN-major
  constexpr uint32_t kIdTV = tc::idesc_bf16_ab(kD, kChunk + 16, 1, 1); // the same with N = 80
  const float sc = P.inv_sqrt_d;
  // keys go round-robin over the CTAs, so the CTAs at work share a query
  // window, whose q, dout and dq rows stay in L2; a key's items are taken in
  // turn, so dK^T, dV^T and v add up in tensor memory over the key's run and
  // go out once at its end
  uint32_t phase = 0;
  bool ok = true;
  for (int key = blockIdx.x; ok && key < ws.n_keys; key += gridDim.x) {
    const int t0 = ws.tile_off[key], t1 = ws.tile_off[key + 1];
    if (t0 == t1) continue;
    const int j = key % P.max_chunks;
    const int bg = key / P.max_chunks / ws.n_win;
    const int g = bg % P.Hkv, b = bg / P.Hkv;
    const int64_t page = page_of(P, b, j);
    if (page < 0) continue;   // the same for every thread of the CTA
    for (int it = t0; it < t1; ++it) {
      const int4 item = ws.items[it];
      const bool run_first = it == t0;
      const bool run_last = it == t1 - 1;
      const int n = item.z - item.y;
      const int row = tid;
      const bool live = row < n;
      int32_t pid = 0;
      int64_t r = 0;
      int nk = 0;
      float wj = 0.f, dl = 0.f;
      if (live) {
        pid = ws.pairs[item.y + row];
        r = pid / P.k;
        const int64_t pos = P.pos0 + (r / P.Hq) % P.L;
        nk = pos / kChunk == j ? (int)(pos - (int64_t)j * kChunk + 1) : kChunk;
        wj = __ldg(wts + pid);
        dl = __ldg(delta + r);
      }
      slm[tid] = __ldg(lmc + (((int64_t)b * P.max_chunks + j) * P.Hkv + g) * kD + tid);
      // ---- the pair's q row into Q (zeros past the item's pairs), K and V
      {
        const uint8_t* src = reinterpret_cast<const uint8_t*>(P.q) + r * (kD * 2);
  #pragma unroll
        for (int c = 0; c < 16; ++c)
          tc::cp_async16(sb + TLay::kQ + tile_at(kRowsT, row, c), src + c * 16, live ? 16u : 0u);
        const uint8_t* kp =
            reinterpret_cast<const uint8_t*>(P.pages) + page_offset(P, page, 0, g, 0) * 2;
        const uint8_t* vp =
            reinterpret_cast<const uint8_t*>(P.pages) + page_offset(P, page, 1, g, 0) * 2;
        for (int x = tid; x < kChunk * 16; x += kThreadsT) {
          const int kr = x >> 4, c = x & 15;
          tc::cp_async16(sb + TLay::kK + tile_at(kChunk, kr, c), kp + kr * (kD * 2) + c * 16, 16u);
          tc::cp_async16(sb + TLay::kV + tile_at(kChunk, kr, c), vp + kr * (kD * 2) + c * 16, 16u);
        }
        tc::cp_async_commit();
        tc::cp_async_wait<0>();
        tc::fence_proxy_async();
      }
      __syncthreads();
      // ---- S = Q K^T
      if (tid == 0) {
        tc::tc_fence_after();
  #pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint64_t a =
              tc::smem_desc(sb + TLay::kQ + (kk >> 2) * (kRowsT * 128) + (kk & 3) * 32, 16, 1024);
          const uint64_t bd =
              tc::smem_desc(sb + TLay::kK + (kk >> 2) * (kChunk * 128) + (kk & 3) * 32, 16, 1024);
          tc::mma_bf16(tmem + kColS, a, bd, kIdS, kk > 0);
        }
        tc::mma_commit(&mma_bar);
      }
      if (!(ok = wait_products(&mma_bar, phase))) break;
      tc::tc_fence_after();
      // ---- this row's P (float32, kept) into the P tile; G = w dout into the G tile
      float p[kChunk];
      {
        uint32_t v[32];
        tc::tmem_ld32(tl + kColS, v);
        tc::tmem_ld_wait();
  #pragma unroll
        for (int x = 0; x < 32; ++x) p[x] = __uint_as_float(v[x]);
        tc::tmem_ld32(tl + kColS + 32, v);
        tc::tmem_ld_wait();
  #pragma unroll
        for (int x = 0; x < 32; ++x) p[32 + x] = __uint_as_float(v[x]);
        float mx = -INFINITY;
  #pragma unroll
        for (int x = 0; x < kChunk; ++x) {
          p[x] = x < nk ? p[x] * sc : -INFINITY;
          mx = fmaxf(mx, p[x]);
        }
        float l = 0.f;
  #pragma unroll
        for (int x = 0; x < kChunk; ++x) {
          p[x] = x < nk ? __expf(p[x] - mx) : 0.f;
          l += p[x];
        }
        const float il = live ? 1.f / l : 0.f;
  #pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint4 u;
          u.x = tc::pack_bf16x2(p[8 * c] * il, p[8 * c + 1] * il);
          u.y = tc::pack_bf16x2(p[8 * c + 2] * il, p[8 * c + 3] * il);
          u.z = tc::pack_bf16x2(p[8 * c + 4] * il, p[8 * c + 5] * il);
          u.w = tc::pack_bf16x2(p[8 * c + 6] * il, p[8 * c + 7] * il);
          *reinterpret_cast<uint4*>(smem + TLay::kP + tc::swz(row, c)) = u;
        }
  #pragma unroll
        for (int x = 0; x < kChunk; ++x) p[x] *= il;
        const uint4* dsrc = reinterpret_cast<const uint4*>(
            reinterpret_cast<const uint8_t*>(dout) + r * (kD * 2));
  #pragma unroll 4
        for (int c = 0; c < 16; ++c) {
          const uint4 d4 = live ? __ldg(dsrc + c) : make_uint4(0, 0, 0, 0);
          uint4 u;
          u.x = tc::pack_bf16x2(wj * bf16_lo(d4.x), wj * bf16_hi(d4.x));
          u.y = tc::pack_bf16x2(wj * bf16_lo(d4.y), wj * bf16_hi(d4.y));
          u.z = tc::pack_bf16x2(wj * bf16_lo(d4.z), wj * bf16_hi(d4.z));
          u.w = tc::pack_bf16x2(wj * bf16_lo(d4.w), wj * bf16_hi(d4.w));
          *reinterpret_cast<uint4*>(smem + TLay::kG + tile_at(kRowsT, row, c)) = u;
        }
      }
      tc::fence_proxy_async();
      tc::tc_fence_before();
      __syncthreads();
      // ---- O = P V (into the O columns) and dP = G V^T (into the S columns)
      if (tid == 0) {
        tc::tc_fence_after();
  #pragma unroll
        for (int kk = 0; kk < kChunk / 16; ++kk) {
          const uint64_t a = tc::smem_desc(sb + TLay::kP + kk * 32, 16, 1024);
          const uint64_t bd = tc::smem_desc(sb + TLay::kV + kk * 2048, kChunk * 128, 1024);
          tc::mma_bf16(tmem + kColO, a, bd, kIdO, kk > 0);
        }
  #pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint64_t a =
              tc::smem_desc(sb + TLay::kG + (kk >> 2) * (kRowsT * 128) + (kk & 3) * 32, 16, 1024);
          const uint64_t bd =
              tc::smem_desc(sb + TLay::kV + (kk >> 2) * (kChunk * 128) + (kk & 3) * 32, 16, 1024);
          tc::mma_bf16(tmem + kColS, a, bd, kIdS, kk > 0);
        }
        tc::mma_commit(&mma_bar);
      }
      if (!(ok = wait_products(&mma_bar, phase))) break;
      tc::tc_fence_after();
      // ---- w dw = G . O (G from its tile); ds = w (dw - delta); dS = P (dP - w dw)
      {
        float go = 0.f;
        uint32_t v[32];
  #pragma unroll
        for (int blk = 0; blk < kD / 32; ++blk) {
          tc::tmem_ld32(tl + kColO + 32 * blk, v);
          tc::tmem_ld_wait();
  #pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint4 g4 =
                *reinterpret_cast<const uint4*>(smem + TLay::kG + tile_at(kRowsT, row, 4 * blk + c));
            go = fmaf(bf16_lo(g4.x), __uint_as_float(v[8 * c + 0]), go);
            go = fmaf(bf16_hi(g4.x), __uint_as_float(v[8 * c + 1]), go);
            go = fmaf(bf16_lo(g4.y), __uint_as_float(v[8 * c + 2]), go);
            go = fmaf(bf16_hi(g4.y), __uint_as_float(v[8 * c + 3]), go);
            go = fmaf(bf16_lo(g4.z), __uint_as_float(v[8 * c + 4]), go);
            go = fmaf(bf16_hi(g4.z), __uint_as_float(v[8 * c + 5]), go);
            go = fmaf(bf16_lo(g4.w), __uint_as_float(v[8 * c + 6]), go);
            go = fmaf(bf16_hi(g4.w), __uint_as_float(v[8 * c + 7]), go);
          }
        }
        sds[row] = live ? go - wj * dl : 0.f;
        srow[row] = live ? (int32_t)r : -1;
  #pragma unroll
        for (int h = 0; h < 2; ++h) {
          tc::tmem_ld32(tl + kColS + 32 * h, v);
          tc::tmem_ld_wait();
  #pragma unroll
          for (int x = 0; x < 32; ++x)
            p[32 * h + x] = p[32 * h + x] * (__uint_as_float(v[x]) - go);
        }
  #pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint4 u;
          u.x = tc::pack_bf16x2(p[8 * c], p[8 * c + 1]);
          u.y = tc::pack_bf16x2(p[8 * c + 2], p[8 * c + 3]);
          u.z = tc::pack_bf16x2(p[8 * c + 4], p[8 * c + 5]);
          u.w = tc::pack_bf16x2(p[8 * c + 6], p[8 * c + 7]);
          *reinterpret_cast<uint4*>(smem + TLay::kS + tc::swz(row, c)) = u;
        }
        // ds as column 0 of the next block (columns 1..15 zero): B of v = Q^T ds
        const uint4 z = make_uint4(0, 0, 0, 0);
        uint4 u0 = z;
        u0.x = tc::pack_bf16x2(sds[row], 0.f);
        *reinterpret_cast<uint4*>(smem + TLay::kS + kPB + tc::swz(row, 0)) = u0;
        *reinterpret_cast<uint4*>(smem + TLay::kS + kPB + tc::swz(row, 1)) = z;
      }
      tc::fence_proxy_async();
      tc::tc_fence_before();
      __syncthreads();
      // ---- dQ = dS K (into the O columns), dK^T = Q^T dS, dV^T = G^T P
      if (tid == 0) {
        tc::tc_fence_after();
  #pragma unroll
        for (int kk = 0; kk < kChunk / 16; ++kk) {
          const uint64_t a = tc::smem_desc(sb + TLay::kS + kk * 32, 16, 1024);
          const uint64_t bd = tc::smem_desc(sb + TLay::kK + kk * 2048, kChunk * 128, 1024);
          tc::mma_bf16(tmem + kColO, a, bd, kIdO, kk > 0);
        }
        // [dK^T | v] = Q^T [dS | ds] (N = 80) and dV^T = G^T P, added to the run's sums
  #pragma unroll
        for (int kk = 0; kk < kRowsT / 16; ++kk) {
          const uint64_t a = tc::smem_desc(sb + TLay::kQ + kk * 2048, kRowsT * 128, 1024);
          const uint64_t bd = tc::smem_desc(sb + TLay::kS + kk * 2048, kRowsT * 128, 1024);
          tc::mma_bf16(tmem + kColDK, a, bd, kIdTV, (kk > 0 || !run_first) ? 1u : 0u);
        }
  #pragma unroll
        for (int kk = 0; kk < kRowsT / 16; ++kk) {
          const uint64_t a = tc::smem_desc(sb + TLay::kG + kk * 2048, kRowsT * 128, 1024);
          const uint64_t bd = tc::smem_desc(sb + TLay::kP + kk * 2048, kRowsT * 128, 1024);
          tc::mma_bf16(tmem + kColDV, a, bd, kIdT, (kk > 0 || !run_first) ? 1u : 0u);
        }
        tc::mma_commit(&mma_bar);
      }
      if (!(ok = wait_products(&mma_bar, phase))) break;
      tc::tc_fence_after();
      // ---- dq row += (dQ + ds lm'_j) / sqrt(d); this thread's element of dK and dV
      {
        // each warp stages its 32 rows, 32 columns at a time, and adds them row
        // by row: 8 lanes cover one row's 128 bytes
        uint32_t v[32];
        const int lr = tid & 31;
        float* stg = reinterpret_cast<float*>(smem + TLay::kStage) + warp * 32 * TLay::kStageLd;
        const float dsr = sds[row];
  #pragma unroll 1
        for (int blk = 0; blk < kD / 32; ++blk) {
          tc::tmem_ld32(tl + kColO + 32 * blk, v);
          tc::tmem_ld_wait();
          const float* lmr = slm + 32 * blk;
  #pragma unroll
          for (int x = 0; x < 32; x += 4)
            *reinterpret_cast<float4*>(stg + lr * TLay::kStageLd + x) =
                make_float4((__uint_as_float(v[x]) + dsr * lmr[x]) * sc,
                            (__uint_as_float(v[x + 1]) + dsr * lmr[x + 1]) * sc,
                            (__uint_as_float(v[x + 2]) + dsr * lmr[x + 2]) * sc,
                            (__uint_as_float(v[x + 3]) + dsr * lmr[x + 3]) * sc);
          __syncwarp();
  #pragma unroll
          for (int pass = 0; pass < 8; ++pass) {
            const int rr = pass * 4 + (lr >> 3), cc = (lr & 7) * 4;
            const int32_t gr = srow[warp * 32 + rr];
            if (gr >= 0)
              tc::red_add_f32x4(dq + (int64_t)gr * kD + 32 * blk + cc,
                                *reinterpret_cast<const float4*>(stg + rr * TLay::kStageLd + cc));
          }
          __syncwarp();
        }
        if (run_last) {
          const int e = tid;   // TMEM lane of dK^T and dV^T = head-dimension element
          float* dk = dpages + page_offset(P, page, 0, g, 0) + e;
          float* dv = dpages + page_offset(P, page, 1, g, 0) + e;
  #pragma unroll
          for (int h = 0; h < 2; ++h) {
            tc::tmem_ld32(tl + kColDK + 32 * h, v);
            tc::tmem_ld_wait();
  #pragma unroll
            for (int x = 0; x < 32; ++x)
              tc::red_add_f32(dk + (32 * h + x) * kD, __uint_as_float(v[x]) * sc);
            tc::tmem_ld32(tl + kColDV + 32 * h, v);
            tc::tmem_ld_wait();
  #pragma unroll
            for (int x = 0; x < 32; ++x) tc::red_add_f32(dv + (32 * h + x) * kD, __uint_as_float(v[x]));
          }
          uint32_t v16[16];
          tc::tmem_ld16(tl + kColV, v16);
          tc::tmem_ld_wait();
          tc::red_add_f32(vchunk + (((int64_t)b * P.max_chunks + j) * P.Hkv + g) * kD + e,
                          __uint_as_float(v16[0]));
        }
      }
      tc::tc_fence_before();
      __syncthreads();   // shared and tensor memory are free for the next item
    }
  }
  if (!ok) {
    // a wait ran out: let the products in flight finish before the memory goes
    if (tid == 0) {
      set_device_error(kErrTimeout);
      tc::mbar_wait(&mma_bar, phase ^ 1u, kDrainLimitNs);
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  if (warp == 0) tc::tmem_dealloc(tmem, kTmemCols);
}

// delta[row] = dout . out, one warp per row.
__global__ void __launch_bounds__(256) delta_kernel(const void* out, const void* dout,
                                                    float* delta, int64_t rows) {
  const int64_t row = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const uint2 o = __ldg(reinterpret_cast<const uint2*>(out) + row * (kD / 4) + lane);
  const uint2 d = __ldg(reinterpret_cast<const uint2*>(dout) + row * (kD / 4) + lane);
  float acc = bf16_lo(o.x) * bf16_lo(d.x);
  acc = fmaf(bf16_hi(o.x), bf16_hi(d.x), acc);
  acc = fmaf(bf16_lo(o.y), bf16_lo(d.y), acc);
  acc = fmaf(bf16_hi(o.y), bf16_hi(d.y), acc);
#pragma unroll
  for (int s = 16; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
  if (lane == 0) delta[row] = acc;
}

// lm'[b][j][g] = lm + (lm B^T) A^T for the chunks j < nvis, one warp each.
__global__ void __launch_bounds__(256) lmc_kernel(Params P, float* lmc, int nvis) {
  __shared__ float sl[8][kD];
  __shared__ float su[8][kMaxRank];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t gw = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (gw >= (int64_t)P.B * nvis * P.Hkv) return;
  const int g = (int)(gw % P.Hkv);
  const int j = (int)((gw / P.Hkv) % nvis);
  const int b = (int)(gw / P.Hkv / nvis);
  const int64_t base = (((int64_t)b * P.max_chunks + j) * P.Hkv + g) * kD;
#pragma unroll
  for (int c = 0; c < kD / 32; ++c) sl[warp][lane + 32 * c] = load_elem(P.landmarks, HILS_BF16, base + lane + 32 * c);
  __syncwarp();
  for (int a = lane; a < P.r; a += 32) {
    float acc = 0.f;
    for (int e = 0; e < kD; ++e) acc = fmaf(sl[warp][e], __ldg(P.Bm + a * kD + e), acc);
    su[warp][a] = acc;
  }
  __syncwarp();
#pragma unroll
  for (int c = 0; c < kD / 32; ++c) {
    const int e = lane + 32 * c;
    float acc = sl[warp][e];
    for (int a = 0; a < P.r; ++a) acc = fmaf(su[warp][a], __ldg(P.A + e * P.r + a), acc);
    lmc[base + e] = acc;
  }
}

// Per chunk row (b, j, g) with its v = sum over the chunk's pairs of ds q:
// dlm += (v + (v A) B) / sqrt(d), and this CTA's share of M = sum of v lm^T
// (thread t keeps row t / 2, half t % 2 of M in registers; mpart[blockIdx.x]
// at the end).  The CTA takes its rows 32 at a time.
constexpr int kPostRows = 32;
__global__ void __launch_bounds__(256) chunk_post_kernel(Params P, const float* vchunk, float* dlm,
                                                         float* mpart, int nvis) {
  extern __shared__ float psm[];
  const int R = P.r, RR = R > 0 ? R : 1;
  float* sA = psm;                        // [kD][R + 1]
  float* sB = sA + kD * (R + 1);          // [R][kD + 1]
  float* sv = sB + R * (kD + 1);          // [kPostRows][kD]
  float* sl = sv + kPostRows * kD;        // [kPostRows][kD]
  float* st = sl + kPostRows * kD;        // [kPostRows][RR]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int x = tid; x < kD * R; x += blockDim.x) sA[(x / R) * (R + 1) + x % R] = P.A[x];
  for (int x = tid; x < R * kD; x += blockDim.x) sB[(x / kD) * (kD + 1) + x % kD] = P.Bm[x];
  const int me = tid >> 1, mf = (tid & 1) * 64;
  float m[64];
#pragma unroll
  for (int f = 0; f < 64; ++f) m[f] = 0.f;
  const float sc = P.inv_sqrt_d;
  const int64_t n_rows = (int64_t)P.B * nvis * P.Hkv;
  for (int64_t r0 = (int64_t)blockIdx.x * kPostRows; r0 < n_rows;
       r0 += (int64_t)gridDim.x * kPostRows) {
    __syncthreads();   // the previous group's rows are no longer read
    for (int x = tid; x < kPostRows * kD; x += blockDim.x) {
      const int lr = x / kD, e = x % kD;
      const int64_t row = r0 + lr;
      float v = 0.f, l = 0.f;
      if (row < n_rows) {
        const int g = (int)(row % P.Hkv);
        const int j = (int)((row / P.Hkv) % nvis);
        const int b = (int)(row / P.Hkv / nvis);
        const int64_t base = (((int64_t)b * P.max_chunks + j) * P.Hkv + g) * kD;
        v = vchunk[base + e];
        l = load_elem(P.landmarks, HILS_BF16, base + e);
      }
      sv[lr * kD + e] = v;
      sl[lr * kD + e] = l;
    }
    __syncthreads();
    // dlm: warp w takes rows 4w .. 4w + 3
    for (int lr = warp * 4; lr < warp * 4 + 4; ++lr) {
      const int64_t row = r0 + lr;
      if (row >= n_rows) break;
      for (int a = lane; a < R; a += 32) {
        float acc = 0.f;
        for (int e = 0; e < kD; ++e) acc = fmaf(sv[lr * kD + e], sA[e * (R + 1) + a], acc);
        st[lr * RR + a] = acc;
      }
      __syncwarp();
      const int g = (int)(row % P.Hkv);
      const int j = (int)((row / P.Hkv) % nvis);
      const int b = (int)(row / P.Hkv / nvis);
      const int64_t base = (((int64_t)b * P.max_chunks + j) * P.Hkv + g) * kD;
#pragma unroll
      for (int c = 0; c < kD / 32; ++c) {
        const int e = lane + 32 * c;
        float acc = sv[lr * kD + e];
        for (int a = 0; a < R; ++a) acc = fmaf(st[lr * RR + a], sB[a * (kD + 1) + e], acc);
        dlm[base + e] += acc * sc;
      }
    }
    // M += v lm^T over the group's rows
    if (R > 0) {
      for (int lr = 0; lr < kPostRows; ++lr) {
        const float ve = sv[lr * kD + me];
        const float* lrow = sl + lr * kD + mf;
#pragma unroll
        for (int f = 0; f < 64; ++f) m[f] = fmaf(ve, lrow[f], m[f]);
      }
    }
  }
  if (R > 0) {
    float* dst = mpart + ((int64_t)blockIdx.x * kD + me) * kD + mf;
#pragma unroll
    for (int f = 0; f < 64; f += 4)
      *reinterpret_cast<float4*>(dst + f) = make_float4(m[f], m[f + 1], m[f + 2], m[f + 3]);
  }
}

// M = sum of the n_cta partials, into mpart[kBackwardMaxCtas].
__global__ void msum_kernel(float* mpart, int n_cta) {
  const int x = blockIdx.x * blockDim.x + threadIdx.x;
  if (x >= kD * kD) return;
  float acc = 0.f;
  for (int c = 0; c < n_cta; ++c) acc += mpart[(int64_t)c * kD * kD + x];
  mpart[(int64_t)kBackwardMaxCtas * kD * kD + x] = acc;
}

// dA += M B^T / sqrt(d) and dB += A^T M / sqrt(d): one thread per entry.
__global__ void dab_kernel(Params P, const float* M, float* dA, float* dB) {
  const int R = P.r;
  const int x = blockIdx.x * blockDim.x + threadIdx.x;
  const float sc = P.inv_sqrt_d;
  if (x < kD * R) {
    const int e = x / R, a = x % R;
    float acc = 0.f;
    for (int f = 0; f < kD; ++f) acc = fmaf(M[e * kD + f], P.Bm[a * kD + f], acc);
    dA[x] += acc * sc;
  } else if (x < 2 * kD * R) {
    const int y = x - kD * R;
    const int a = y / kD, f = y % kD;
    float acc = 0.f;
    for (int e = 0; e < kD; ++e) acc = fmaf(P.A[e * R + a], M[e * kD + f], acc);
    dB[y] += acc * sc;
  }
}

}  // namespace

cudaError_t launch_backward_tc(const Params& P, const int32_t* idx, const float* w,
                               const void* out, const void* dout, float* dq, float* dpages,
                               float* dlm, float* dA, float* dB, const BackwardWs& ws,
                               cudaStream_t s) {
  (void)idx;
  cudaError_t e;
  const int64_t rows = (int64_t)P.B * P.L * P.Hq;
  const int nvis = (int)((P.pos0 + P.L - 1) / kChunk + 1 < P.max_chunks
                             ? (P.pos0 + P.L - 1) / kChunk + 1
                             : P.max_chunks);
  {
    HILS_PROFILE("backward.prepare", s);
    delta_kernel<<<(unsigned)((rows * 32 + 255) / 256), 256, 0, s>>>(out, dout, ws.delta, rows);
    const int64_t warps = (int64_t)P.B * nvis * P.Hkv;
    lmc_kernel<<<(unsigned)((warps * 32 + 255) / 256), 256, 0, s>>>(P, ws.lmc, nvis);
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const size_t smem = TLay::kBytes + 1024;   // + alignment slack
  if ((e = set_smem(attn_bwd_tc_kernel, smem)) != cudaSuccess) return e;
  int dev = 0, n_sm = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return e;
  const size_t vbytes = sizeof(float) * (size_t)P.B * P.max_chunks * P.Hkv * kD;
  if ((e = cudaMemsetAsync(ws.vchunk, 0, vbytes, s)) != cudaSuccess) return e;
  const int64_t grid = ws.bk.n_keys < n_sm ? ws.bk.n_keys : n_sm;
  {
    HILS_PROFILE("backward.attention", s);
    attn_bwd_tc_kernel<<<(unsigned)(grid > 0 ? grid : 1), kThreadsT, smem, s>>>(
        P, ws.bk, w, dout, ws.delta, ws.lmc, ws.vchunk, dq, dpages);
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int64_t n_rows = (int64_t)P.B * nvis * P.Hkv;
  const int64_t groups = (n_rows + kPostRows - 1) / kPostRows;
  const int n_cta = (int)(groups < kBackwardMaxCtas ? groups : kBackwardMaxCtas);
  const size_t psm = sizeof(float) * ((size_t)kD * (P.r + 1) + (size_t)P.r * (kD + 1) +
                                      2 * kPostRows * kD + kPostRows * (P.r > 0 ? P.r : 1));
  if ((e = set_smem(chunk_post_kernel, psm)) != cudaSuccess) return e;
  {
    HILS_PROFILE("backward.landmarks", s);
    chunk_post_kernel<<<(unsigned)(n_cta > 0 ? n_cta : 1), 256, psm, s>>>(P, ws.vchunk, dlm,
                                                                        ws.mpart, nvis);
    if (P.r > 0) {
      msum_kernel<<<(kD * kD + 255) / 256, 256, 0, s>>>(ws.mpart, n_cta > 0 ? n_cta : 1);
      dab_kernel<<<(unsigned)((2 * kD * P.r + 255) / 256), 256, 0, s>>>(
          P, ws.mpart + (int64_t)kBackwardMaxCtas * kD * kD, dA, dB);
    }
  }
  return cudaGetLastError();
}

}  // namespace hils
