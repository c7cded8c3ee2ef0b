// Attention part of the prefill backward on the tensor cores (bf16 storage,
// head_dim 128).  Each work item of the key-major buckets (up to 128 pairs of
// one chunk and KV head) is one tile of M = 128 rows, one per pair.  With Q
// the pairs' query rows, G = w dout their weighted output gradients, and K, V
// the chunk's keys and values:
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
// does the element-wise work, and thread 0 issues the products.  The kernel is
// persistent: one CTA per SM walks the items.  dq and the pool's gradient
// receive float32 additions in L2.  The same quantities on CUDA cores, for
// the other configurations, are in backward.cu.
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
  static constexpr uint32_t kS = kP + kPB;
  static constexpr uint32_t kBytes = kS + kPB;       // 128 KB
};
constexpr uint32_t kColS = 0, kColO = 64, kColDK = 192, kColDV = 256, kTmemCols = 512;

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
    attn_bwd_tc_kernel(Params P, PrefillWs ws, const float* wts, const void* dout, float* dq,
                       float* dpages, float* dw) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t mma_bar;
  __shared__ uint32_t tmem_sh;
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
  const float sc = P.inv_sqrt_d;
  const int n_items = ws.tile_off[ws.n_keys];
  uint32_t phase = 0;
  bool ok = true;
  for (int it = blockIdx.x; ok && it < n_items; it += gridDim.x) {
    const int4 item = ws.items[it];
    const int key = item.x;
    const int j = key % P.max_chunks;
    const int bg = key / P.max_chunks / ws.n_win;
    const int g = bg % P.Hkv, b = bg / P.Hkv;
    const int64_t page = page_of(P, b, j);
    if (page < 0) continue;   // the same for every thread of the CTA
    const int n = item.z - item.y;
    const int row = tid;
    const bool live = row < n;
    int32_t pid = 0;
    int64_t r = 0;
    int nk = 0;
    float wj = 0.f;
    if (live) {
      pid = ws.pairs[item.y + row];
      r = pid / P.k;
      const int64_t pos = P.pos0 + (r / P.Hq) % P.L;
      nk = pos / kChunk == j ? (int)(pos - (int64_t)j * kChunk + 1) : kChunk;
      wj = __ldg(wts + pid);
    }
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
    // ---- dw = dout . O; dS = P (dP - w dw) into the dS tile
    {
      const uint4* dsrc = reinterpret_cast<const uint4*>(
          reinterpret_cast<const uint8_t*>(dout) + r * (kD * 2));
      float dwp = 0.f;
      uint32_t v[32];
#pragma unroll
      for (int blk = 0; blk < kD / 32; ++blk) {
        tc::tmem_ld32(tl + kColO + 32 * blk, v);
        tc::tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint4 d4 = live ? __ldg(dsrc + 4 * blk + c) : make_uint4(0, 0, 0, 0);
          dwp = fmaf(bf16_lo(d4.x), __uint_as_float(v[8 * c + 0]), dwp);
          dwp = fmaf(bf16_hi(d4.x), __uint_as_float(v[8 * c + 1]), dwp);
          dwp = fmaf(bf16_lo(d4.y), __uint_as_float(v[8 * c + 2]), dwp);
          dwp = fmaf(bf16_hi(d4.y), __uint_as_float(v[8 * c + 3]), dwp);
          dwp = fmaf(bf16_lo(d4.z), __uint_as_float(v[8 * c + 4]), dwp);
          dwp = fmaf(bf16_hi(d4.z), __uint_as_float(v[8 * c + 5]), dwp);
          dwp = fmaf(bf16_lo(d4.w), __uint_as_float(v[8 * c + 6]), dwp);
          dwp = fmaf(bf16_hi(d4.w), __uint_as_float(v[8 * c + 7]), dwp);
        }
      }
      if (live) dw[pid] = dwp;
      const float go = wj * dwp;
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
#pragma unroll
      for (int kk = 0; kk < kRowsT / 16; ++kk) {
        const uint64_t a = tc::smem_desc(sb + TLay::kQ + kk * 2048, kRowsT * 128, 1024);
        const uint64_t bd = tc::smem_desc(sb + TLay::kS + kk * 2048, kRowsT * 128, 1024);
        tc::mma_bf16(tmem + kColDK, a, bd, kIdT, kk > 0);
      }
#pragma unroll
      for (int kk = 0; kk < kRowsT / 16; ++kk) {
        const uint64_t a = tc::smem_desc(sb + TLay::kG + kk * 2048, kRowsT * 128, 1024);
        const uint64_t bd = tc::smem_desc(sb + TLay::kP + kk * 2048, kRowsT * 128, 1024);
        tc::mma_bf16(tmem + kColDV, a, bd, kIdT, kk > 0);
      }
      tc::mma_commit(&mma_bar);
    }
    if (!(ok = wait_products(&mma_bar, phase))) break;
    tc::tc_fence_after();
    // ---- dq row += dQ / sqrt(d); this thread's head-dimension element of dK and dV
    {
      uint32_t v[32];
#pragma unroll
      for (int blk = 0; blk < kD / 32; ++blk) {
        tc::tmem_ld32(tl + kColO + 32 * blk, v);
        tc::tmem_ld_wait();
        if (live) {
          float4* dst = reinterpret_cast<float4*>(dq + r * kD + 32 * blk);
#pragma unroll
          for (int x = 0; x < 8; ++x)
            atomicAdd(dst + x, make_float4(__uint_as_float(v[4 * x]) * sc,
                                           __uint_as_float(v[4 * x + 1]) * sc,
                                           __uint_as_float(v[4 * x + 2]) * sc,
                                           __uint_as_float(v[4 * x + 3]) * sc));
        }
      }
      const int e = tid;   // TMEM lane of dK^T and dV^T = head-dimension element
      float* dk = dpages + page_offset(P, page, 0, g, 0) + e;
      float* dv = dpages + page_offset(P, page, 1, g, 0) + e;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        tc::tmem_ld32(tl + kColDK + 32 * h, v);
        tc::tmem_ld_wait();
#pragma unroll
        for (int x = 0; x < 32; ++x) atomicAdd(dk + (32 * h + x) * kD, __uint_as_float(v[x]) * sc);
        tc::tmem_ld32(tl + kColDV + 32 * h, v);
        tc::tmem_ld_wait();
#pragma unroll
        for (int x = 0; x < 32; ++x) atomicAdd(dv + (32 * h + x) * kD, __uint_as_float(v[x]));
      }
    }
    tc::tc_fence_before();
    __syncthreads();   // shared and tensor memory are free for the next item
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

}  // namespace

cudaError_t launch_attn_bwd_tc(const Params& P, const PrefillWs& ws, const float* w,
                               const void* dout, float* dq, float* dpages, float* dw,
                               cudaStream_t s) {
  const size_t smem = TLay::kBytes + 1024;   // + alignment slack
  cudaError_t e = set_smem(attn_bwd_tc_kernel, smem);
  if (e != cudaSuccess) return e;
  int dev = 0, n_sm = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return e;
  const int64_t grid = ws.max_tiles < n_sm ? ws.max_tiles : n_sm;
  HILS_PROFILE("backward.attention", s);
  attn_bwd_tc_kernel<<<(unsigned)(grid > 0 ? grid : 1), kThreadsT, smem, s>>>(P, ws, w, dout, dq,
                                                                            dpages, dw);
  return cudaGetLastError();
}

}  // namespace hils
