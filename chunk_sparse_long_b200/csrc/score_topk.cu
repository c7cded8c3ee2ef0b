// hils_score (a1 + a2 materialised) and hils_topk (a3 + a4 on given scores).
// One warp per query row; meant for tests and small inputs -- the prefill and
// decode paths never materialise the score matrix.
#include <cfloat>

#include "hils_common.cuh"

namespace hils {

__device__ int g_device_error = 0;
__constant__ uint64_t g_wait_limit_ns = kDrainLimitNs;

namespace {

constexpr int kWarpsPerBlock = 8;

// q~ = q + (q A) B for one row, computed by one warp into shared memory.
// qs: [d] raw q (already loaded), ts: [r] scratch, qt: [d] result.
__device__ void warp_calibrate(const Params& P, const float* qs, float* ts, float* qt) {
  const int lane = threadIdx.x & 31;
  for (int a = lane; a < P.r; a += 32) {
    float acc = 0.f;
    for (int e = 0; e < P.d; ++e) acc = fmaf(qs[e], P.A[e * P.r + a], acc);
    ts[a] = acc;
  }
  __syncwarp();
  for (int e = lane; e < P.d; e += 32) {
    float acc = 0.f;
    for (int a = 0; a < P.r; ++a) acc = fmaf(ts[a], P.Bm[a * P.d + e], acc);
    qt[e] = qs[e] + acc;
  }
  __syncwarp();
}

__global__ void score_kernel(Params P, float* scores, int n_cols) {
  __shared__ float sq[kWarpsPerBlock][128];
  __shared__ float sqt[kWarpsPerBlock][128];
  __shared__ float st[kWarpsPerBlock][kMaxRank];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t rows = (int64_t)P.B * P.L * P.Hq;
  const int64_t r = (int64_t)blockIdx.x * kWarpsPerBlock + warp;
  if (r >= rows) return;
  const int h = (int)(r % P.Hq);
  const int64_t i = (r / P.Hq) % P.L;
  const int b = (int)(r / ((int64_t)P.Hq * P.L));
  const int g = h / P.group;
  const int64_t pos = P.pos0 + i;
  const int64_t own = pos / kChunk;
  for (int e = lane; e < P.d; e += 32) sq[warp][e] = load_elem(P.q, P.dtype, r * P.d + e);
  __syncwarp();
  warp_calibrate(P, sq[warp], st[warp], sqt[warp]);
  for (int64_t j = lane; j < n_cols; j += 32) {
    float s = -INFINITY;
    if (j <= own) {
      const int64_t base = (((int64_t)b * P.max_chunks + j) * P.Hkv + g) * P.d;
      float acc = 0.f;
      for (int e = 0; e < P.d; e += 8) {
        float v[8];
        load8(P.landmarks, P.dtype, base + e, v);
#pragma unroll
        for (int u = 0; u < 8; ++u) acc = fmaf(sqt[warp][e + u], v[u], acc);
      }
      s = acc * P.inv_sqrt_d;
    }
    scores[r * n_cols + j] = s;
  }
}

// True when (sa, ja) comes before (sb, jb) in (score desc, index asc) order.
__device__ __forceinline__ bool before(float sa, int ja, float sb, int jb) {
  return sa > sb || (sa == sb && ja < jb);
}

__global__ void topk_kernel(Params P, const float* scores, int n_cols, int32_t* idx, float* w) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t rows = (int64_t)P.B * P.L * P.Hq;
  const int64_t r = (int64_t)blockIdx.x * kWarpsPerBlock + warp;
  if (r >= rows) return;
  const int64_t i = (r / P.Hq) % P.L;
  int64_t own = (P.pos0 + i) / kChunk;
  if (own > n_cols - 1) own = n_cols - 1;
  const float* s = scores + r * n_cols;
  // slot a of the result lives in lane a
  float my_s = -INFINITY;
  int my_j = -1;
  if (lane == 0) {
    my_s = s[own];
    my_j = (int)own;
  }
  float last_s = INFINITY;
  int last_j = -1;
  int n = 1;
  for (int slot = 1; slot < P.k && slot <= own; ++slot) {
    // best candidate strictly after (last_s, last_j) in the order
    float bs = -INFINITY;
    int bj = INT32_MAX;
    for (int64_t j = lane; j < own; j += 32) {
      float v = s[j];
      if (before(last_s, last_j, v, (int)j) && (bj == INT32_MAX || before(v, (int)j, bs, bj))) {
        bs = v;
        bj = (int)j;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      float os = __shfl_xor_sync(0xffffffffu, bs, o);
      int oj = __shfl_xor_sync(0xffffffffu, bj, o);
      if (oj != INT32_MAX && (bj == INT32_MAX || before(os, oj, bs, bj))) {
        bs = os;
        bj = oj;
      }
    }
    if (lane == slot) {
      my_s = bs;
      my_j = bj;
    }
    last_s = bs;
    last_j = bj;
    ++n;
  }
  // fusion weights: softmax over the n selected scores
  float m = lane < n ? my_s : -INFINITY;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float e = lane < n ? __expf(my_s - m) : 0.f;
  float z = e;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
  if (lane < P.k) {
    idx[r * P.k + lane] = lane < n ? my_j : -1;
    w[r * P.k + lane] = lane < n ? e / z : 0.f;
  }
}

}  // namespace

cudaError_t launch_score(const Params& P, float* scores, int n_cols, cudaStream_t s) {
  const int64_t rows = (int64_t)P.B * P.L * P.Hq;
  if (rows == 0) return cudaSuccess;
  const int64_t blocks = (rows + kWarpsPerBlock - 1) / kWarpsPerBlock;
  HILS_PROFILE("score", s);
  score_kernel<<<(unsigned)blocks, kWarpsPerBlock * 32, 0, s>>>(P, scores, n_cols);
  return cudaGetLastError();
}

cudaError_t launch_topk(const Params& P, const float* scores, int n_cols, int32_t* idx, float* w,
                        cudaStream_t s) {
  const int64_t rows = (int64_t)P.B * P.L * P.Hq;
  if (rows == 0) return cudaSuccess;
  const int64_t blocks = (rows + kWarpsPerBlock - 1) / kWarpsPerBlock;
  HILS_PROFILE("topk", s);
  topk_kernel<<<(unsigned)blocks, kWarpsPerBlock * 32, 0, s>>>(P, scores, n_cols, idx, w);
  return cudaGetLastError();
}

}  // namespace hils
