// Prefill per-chunk attention (a5) and fused merge (a6) on the 5th-generation
// tensor cores (tcgen05, TMEM accumulators), bf16 inputs.
//
// Work is key-major: the (row, slot) pairs are bucketed by (sequence, KV head,
// query window, chunk) and a work item is up to kItemPairs pairs of one
// bucket, so the chunk's 64 x d K and V tiles are staged in shared memory once
// per item and shared by up to four 128-row tiles.  One persistent CTA per SM
// runs a warp-specialised pipeline over its items' tiles:
//
//   warps 0-3 (producers)  take items in a fixed order; per item copy K
//       and V into one of two buffers, per tile gather the 128 pairs' query
//       rows (cp.async, 16 B; warp w the rows 32w ..) into one of NS
//       128-byte-swizzled K-major stages and publish the tile (rows, causal
//       key counts) on the stage's barrier.
//   warp 4 (MMA)  one thread polls the barriers and issues, as soon as each
//       is ready, S = Q K^T (M=128, N=64) into the TMEM S buffer of the
//       tile's group, or O = P V of a tile whose softmax is done.  V is read
//       MN-major with one extra 64-column block whose first column is all
//       ones (N = d + 16), so column d of O is l = sum of the bf16 P row,
//       summed by the tensor core in float32.
//   warps 5-8, 9-12 (two groups, even / odd tiles)  thread t of a group owns
//       tile row t (TMEM lane t): softmax of its 64 logits, keys after the
//       query masked in the own chunk, P (bf16) written over the consumed Q
//       stage; then O / l -> bf16 into the same stage, which is handed to
//       the store warp, and the group moves on to its next tile.
//   warps 13, 14 (stores)  warp 13 + g serves group g: one thread writes each
//       staged tile with a single bulk copy, waits until the copy has read
//       the stage, and only then frees the stage for the producers.  The
//       groups never wait for their stores.
//
// Partials are stored in bucket order, one row of d bf16 per pair (16-byte
// chunk c of the row at chunk slot c ^ (position & 7)); merge_kernel then sums
// each query row's k partials times the fusion weights in float32, slot order
// (deterministic), and writes the output row.
#include <cfloat>

#include "hils_common.cuh"
#include "tc_common.cuh"

namespace hils {
namespace {

constexpr int kRows = 128;          // pairs per MMA tile (M)
constexpr int kProducers = 4;       // producer warps
constexpr int kMmaWarp = kProducers;
constexpr int kWarps = kProducers + 1 + 8 + 2;  // producers, MMA, two groups of four, stores
constexpr int kStoreWarp = kProducers + 1 + 8;  // first of the two store warps
constexpr int kThreads = kWarps * 32;

template <int D>
struct AttnLayout {
  static constexpr int NS = 4;                          // query stages
  static constexpr uint32_t kQBytes = kRows * D * 2;   // one query tile
  static constexpr uint32_t kKVBytes = kChunk * D * 2; // one K (or V) tile
  static constexpr uint32_t kBlkBytes = kChunk * 128;  // one 64-column block of a K/V tile
  static constexpr uint32_t kVBuf = kKVBytes + kBlkBytes;  // V tile + the ones block
  static constexpr uint32_t kQ = 0;                    // NS stages
  static constexpr uint32_t kK = NS * kQBytes;         // two K buffers
  static constexpr uint32_t kV = kK + 2 * kKVBytes;    // two V buffers (+ ones blocks)
  static constexpr uint32_t kEnd = kV + 2 * kVBuf;
  static constexpr uint32_t kSmem = kEnd + 1024;       // + slack for 1024-byte alignment
  static constexpr int kNO = D + 16;                   // O columns: d values and l
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kTmemS = 0;                // two S buffers of 64 columns
  static constexpr uint32_t kTmemO = 2 * kChunk;       // two O buffers of kNO columns
};

struct TileDesc {
  int32_t tile_base;  // bucket position of the tile's row 0
  int32_t n_valid;    // rows in use
  int32_t kb;         // K/V buffer
  int32_t kv_phase;   // parity of that buffer's fill
  int32_t first, last, end;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(Params P, PrefillWs ws) {
  using Lay = AttnLayout<D>;
  constexpr int NS = Lay::NS;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t q_full[NS], q_empty[NS], kv_full[2], kv_empty[2];
  __shared__ uint64_t s_full[2], sm_done[2], o_full[2], o_free[2];
  __shared__ TileDesc desc[NS];
  __shared__ uint64_t staged[NS];         // a group has written the stage's output rows
  __shared__ int64_t st_dst[NS];          // their byte offset in the partials
  __shared__ uint32_t st_bytes[NS];       // and size; 0 marks the group's end
  __shared__ uint8_t meta_nk[NS][kRows];  // keys visible to it (64, or fewer in the own chunk)
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~(uintptr_t)1023);
  const uint32_t sbase = tc::smem_u32(smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int x = 0; x < NS; ++x) {
      tc::mbar_init(&q_full[x], 64 * kProducers);   // a cp.async and a plain arrival per producer
      tc::mbar_init(&q_empty[x], 1);
      tc::mbar_init(&staged[x], 1);
    }
    for (int x = 0; x < 2; ++x) {
      tc::mbar_init(&kv_full[x], 32 * kProducers);
      tc::mbar_init(&kv_empty[x], 1);
      tc::mbar_init(&s_full[x], 1);
      tc::mbar_init(&sm_done[x], 128);
      tc::mbar_init(&o_full[x], 1);
      tc::mbar_init(&o_free[x], 128);
    }
    tc::fence_mbar_init();
    abort_sh = 0;
  }
  if (warp == kMmaWarp) {
    tc::tmem_alloc(&tmem_base_sh, Lay::kTmemCols);
    tc::tmem_relinquish();
  }
  // the ones block after each V tile: element 0 of every key row is 1.0 (bf16)
  for (int x = tid; x < 2 * (int)Lay::kBlkBytes / 16; x += kThreads) {
    const int buf = x / (Lay::kBlkBytes / 16), y = x % (Lay::kBlkBytes / 16);
    const int s = y >> 3, c = y & 7;
    uint8_t* blk = smem + Lay::kV + buf * Lay::kVBuf + Lay::kKVBytes;
    *reinterpret_cast<uint4*>(blk + tc::swz(s, c)) = make_uint4(c == 0 ? 0x3F80u : 0u, 0u, 0u, 0u);
  }
  tc::fence_proxy_async();
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  const int n_items = ws.tile_off[ws.n_keys];

  if (warp < kProducers) {
    // --------------------------------------------------------------- producers
    // Items are taken in a fixed order (blockIdx.x, + gridDim.x, ...), so the
    // dependent loads are issued ahead of their use: the (key, pair range) of
    // the item after next, the page of the next item's chunk, and the pair id
    // of this thread's row in the next tile.
    constexpr int CPR = D / 8;       // 16-byte chunks per row
    constexpr int RPI = 32 / CPR;    // rows per warp-wide copy instruction
    const int ptid = tid;            // 0 .. 32 * kProducers - 1
    const int my_row = warp * 32 + lane;
    const int stride = gridDim.x;
    auto item_info = [&](int it) {
      return it < n_items ? ws.items[it] : make_int4(0, 0, 0, 0);
    };
    // block-table entry of the chunk of item `it` (raw; checked when used)
    auto raw_page = [&](int it, const int4& inf) -> int32_t {
      if (it >= n_items) return -1;
      const int j = inf.x % P.max_chunks;
      const int b = inf.x / P.max_chunks / ws.n_win / P.Hkv;
      return P.block_table[(int64_t)b * P.max_chunks + j];
    };
    int item = blockIdx.x;
    int4 info = item_info(item);
    int4 info_next = item_info(item + stride);
    int32_t page_raw = raw_page(item, info);
    // (query row, position) of this thread's row in the next tile; x = -1: unused row
    int2 pi_next = (item < n_items && info.y + my_row < info.z) ? ws.pinfo[info.y + my_row]
                                                                : make_int2(-1, 0);
    int n = 0;
    bool ok = true;
    for (int item_idx = 0;; ++item_idx) {
      // every producer thread takes the same decision here
      if (tc::named_barrier_or(3, 32 * kProducers, !ok || abort_sh != 0)) {
        ok = false;
        break;
      }
      if (item >= n_items) break;
      const int next_item = item + stride;
      const int4 info_after = item_info(next_item + stride);
      const int32_t page_raw_next = raw_page(next_item, info_next);
      const int key = info.x;
      const int j = key % P.max_chunks;
      const int bg = key / P.max_chunks / ws.n_win;
      const int g = bg % P.Hkv;
      const int p0 = info.y, p1 = info.z;
      const int nt = (p1 - p0 + kRows - 1) / kRows;
      const int kb = item_idx & 1;
      if (item_idx >= 2 && !tc::mbar_wait(&kv_empty[kb], ((item_idx >> 1) - 1) & 1)) {
        ok = false;
        continue;
      }
      {
        int64_t page = page_raw;
        if (page < 0 || page >= P.num_pages) {
          set_device_error(kErrPage);
          page = -1;
        }
        const uint16_t* kp = reinterpret_cast<const uint16_t*>(P.pages) +
                             (page >= 0 ? page_offset(P, page, 0, g, 0) : 0);
        const uint16_t* vp = reinterpret_cast<const uint16_t*>(P.pages) +
                             (page >= 0 ? page_offset(P, page, 1, g, 0) : 0);
        const uint32_t bytes = page >= 0 ? 16u : 0u;
        const uint32_t kdst = sbase + Lay::kK + kb * Lay::kKVBytes;
        const uint32_t vdst = sbase + Lay::kV + kb * Lay::kVBuf;
        for (int x = ptid; x < kChunk * CPR; x += 32 * kProducers) {
          const int s = x / CPR, c = x % CPR;
          const uint32_t off = (uint32_t)(c >> 3) * (kChunk * 128) + tc::swz(s, c & 7);
          tc::cp_async16(kdst + off, kp + s * D + c * 8, bytes);
          tc::cp_async16(vdst + off, vp + s * D + c * 8, bytes);
        }
        tc::cp_async_mbar_arrive(&kv_full[kb]);
      }
      for (int t = 0; t < nt && ok; ++t, ++n) {
        const int st = n % NS;
        if (n >= NS && !tc::mbar_wait(&q_empty[st], ((n / NS) - 1) & 1)) {
          ok = false;
          break;
        }
        const int tile_base = p0 + t * kRows;
        const int nv = min(kRows, p1 - tile_base);
        const int2 pi = pi_next;
        // this row's pair in the next tile: of this item, or the first tile of the next
        {
          int pn, pend;
          if (t + 1 < nt) {
            pn = tile_base + kRows + my_row;
            pend = p1;
          } else {
            pn = info_next.y + my_row;
            pend = next_item < n_items ? info_next.z : 0;
          }
          pi_next = pn < pend ? ws.pinfo[pn] : make_int2(-1, 0);
        }
        const int32_t my_r = pi.x;
        {
          int nk = kChunk;
          if (my_r >= 0) {
            const int64_t pos = P.pos0 + pi.y;
            if (pos / kChunk == j) nk = (int)(pos - (int64_t)j * kChunk + 1);
          }
          meta_nk[st][my_row] = (uint8_t)nk;
        }
        const uint32_t qdst = sbase + Lay::kQ + st * Lay::kQBytes;
#pragma unroll
        for (int it = 0; it < 32 / RPI; ++it) {
          const int row = warp * 32 + it * RPI + lane / CPR, c = lane % CPR;
          const int32_t r = __shfl_sync(0xffffffffu, my_r, it * RPI + lane / CPR);
          const uint16_t* src =
              reinterpret_cast<const uint16_t*>(P.q) + (int64_t)(r >= 0 ? r : 0) * D + c * 8;
          tc::cp_async16(qdst + (uint32_t)(c >> 3) * (kRows * 128) + tc::swz(row, c & 7), src,
                         r >= 0 ? 16u : 0u);
        }
        if (ptid == 0) {
          TileDesc d;
          d.tile_base = tile_base;
          d.n_valid = nv;
          d.kb = kb;
          d.kv_phase = (item_idx >> 1) & 1;
          d.first = t == 0;
          d.last = t == nt - 1;
          d.end = 0;
          desc[st] = d;
        }
        tc::cp_async_mbar_arrive(&q_full[st]);
        tc::mbar_arrive(&q_full[st]);
      }
      item = next_item;
      info = info_next;
      info_next = info_after;
      page_raw = page_raw_next;
    }
    // two end markers: one for each group
    for (int e = 0; e < 2 && ok; ++e, ++n) {
      const int st = n % NS;
      if (n >= NS && !tc::mbar_wait(&q_empty[st], ((n / NS) - 1) & 1)) {
        ok = false;
        break;
      }
      if (ptid == 0) {
        TileDesc d{};
        d.end = 1;
        desc[st] = d;
      }
      tc::cp_async_mbar_arrive(&q_full[st]);
      tc::mbar_arrive(&q_full[st]);
    }
    if (!ok) abort_sh = 1;
    tc::cp_async_wait<0>();
  } else if (warp == kMmaWarp) {
    // -------------------------------------------------------------------- MMA
    if (lane == 0) {
      constexpr uint32_t kIdS = tc::idesc_bf16(kRows, kChunk, 0);
      constexpr uint32_t kIdO = tc::idesc_bf16(kRows, Lay::kNO, 1);
      int ns = 0, np = 0;        // next tile to issue S for / P V for
      bool s_done = false;
      uint64_t t_idle = 0;
      uint32_t idle = 0;
      for (;;) {
        bool progress = false;
        // O = P V of tile np once its softmax is done and its O buffer is free
        if (np < ns) {
          const int wg = np & 1;
          if (tc::mbar_try_wait(&sm_done[wg], (np >> 1) & 1) &&
              (np < 2 || tc::mbar_try_wait(&o_free[wg], ((np >> 1) - 1) & 1))) {
            tc::tc_fence_after();
            const TileDesc dm = desc[np % NS];
            const uint32_t pst = sbase + Lay::kQ + (np % NS) * Lay::kQBytes;
            const uint32_t vb = sbase + Lay::kV + dm.kb * Lay::kVBuf;
#pragma unroll
            for (int kk = 0; kk < kChunk / 16; ++kk) {
              const uint64_t a = tc::smem_desc(pst + kk * 32, 16, 1024);
              const uint64_t bd = tc::smem_desc(vb + kk * 2048, kChunk * 128, 1024);
              tc::mma_bf16(tmem + Lay::kTmemO + wg * Lay::kNO, a, bd, kIdO, kk > 0);
            }
            tc::mma_commit(&o_full[wg]);
            if (dm.last) tc::mma_commit(&kv_empty[dm.kb]);
            ++np;
            progress = true;
          }
        }
        // S = Q K^T of tile ns once it is gathered and its S buffer is free
        if (!s_done) {
          const int st = ns % NS, wg = ns & 1;
          if (tc::mbar_try_wait(&q_full[st], (ns / NS) & 1)) {
            const TileDesc d = desc[st];
            if (d.end) {
              s_done = true;
            } else if ((!d.first || tc::mbar_try_wait(&kv_full[d.kb], d.kv_phase)) &&
                       (ns < 2 || tc::mbar_try_wait(&sm_done[wg], ((ns >> 1) - 1) & 1))) {
              tc::tc_fence_after();
              const uint32_t qst = sbase + Lay::kQ + st * Lay::kQBytes;
              const uint32_t kbuf = sbase + Lay::kK + d.kb * Lay::kKVBytes;
#pragma unroll
              for (int kk = 0; kk < D / 16; ++kk) {
                const uint64_t a = tc::smem_desc(qst + (kk >> 2) * (kRows * 128) + (kk & 3) * 32, 16, 1024);
                const uint64_t bd = tc::smem_desc(kbuf + (kk >> 2) * (kChunk * 128) + (kk & 3) * 32, 16, 1024);
                tc::mma_bf16(tmem + Lay::kTmemS + wg * kChunk, a, bd, kIdS, kk > 0);
              }
              tc::mma_commit(&s_full[wg]);
              ++ns;
              progress = true;
            }
          }
        }
        if (s_done && np == ns) break;
        if (progress || abort_sh) {
          idle = 0;
          if (abort_sh) break;
        } else if ((++idle & 255u) == 0) {
          const uint64_t now = tc::globaltimer_ns();
          if (idle == 256) t_idle = now;
          else if (now - t_idle > 2000000000ull) {
            abort_sh = 1;
            break;
          }
        }
      }
    }
    __syncwarp();
  } else if (warp >= kStoreWarp) {
    // ------------------------------------------------------------------ stores
    // warp kStoreWarp + g takes group g's tiles (n = g, g + 2, ..): stages
    // g, g + 2 (mod NS)
    if (lane == 0) {
      bool ok = true;
      for (int n = warp - kStoreWarp;; n += 2) {
        const int st = n % NS;
        if (!tc::mbar_wait_sleep(&staged[st], (n / NS) & 1)) {
          ok = false;
          break;
        }
        const uint32_t bytes = st_bytes[st];
        if (bytes == 0) break;
        tc::bulk_s2g(reinterpret_cast<uint8_t*>(ws.partial) + st_dst[st],
                     sbase + Lay::kQ + st * Lay::kQBytes, bytes);
        tc::bulk_commit();
        tc::bulk_wait_read();
        tc::mbar_arrive(&q_empty[st]);
      }
      if (!ok) abort_sh = 1;
      tc::bulk_wait_all();
    }
    __syncwarp();
  } else {
    // ---------------------------------------------- softmax + epilogue groups
    const int wg = (warp - kMmaWarp - 1) >> 2;
    const int row = ((warp & 3) << 5) + lane;            // TMEM lane of this warp's quarter
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const float scale_log2 = P.inv_sqrt_d * 1.4426950408889634f;
    bool ok = true;
    for (int n = wg, u = 0;; n += 2, ++u) {
      const int st = n % NS;
      bool bad = !tc::warp_wait(&q_full[st], (n / NS) & 1);
      const TileDesc d = desc[st];
      // the group leaves together or not at all (its named barrier below)
      if (tc::named_barrier_or(1 + wg, 128, bad)) {
        ok = false;
        break;
      }
      if (d.end) {
        if (row == 0) {
          st_bytes[st] = 0;
          tc::mbar_arrive(&staged[st]);
        }
        break;
      }
      const int nk = meta_nk[st][row];
      uint8_t* stage = smem + Lay::kQ + st * Lay::kQBytes;
      bad = !tc::warp_wait(&s_full[wg], u & 1);
      if (!bad) {
        tc::tc_fence_after();
        uint32_t sr[64];
        {
          uint32_t a[32], c[32];
          tc::tmem_ld32(tmem + lane_off + Lay::kTmemS + wg * kChunk, a);
          tc::tmem_ld32(tmem + lane_off + Lay::kTmemS + wg * kChunk + 32, c);
          tc::tmem_ld_wait();
#pragma unroll
          for (int x = 0; x < 32; ++x) {
            sr[x] = a[x];
            sr[32 + x] = c[x];
          }
        }
        // keys after the query exist only in the own chunk: a warp-uniform branch
        const bool masked = !__all_sync(0xffffffffu, nk == kChunk);
        float m = -INFINITY;
        if (!masked) {
#pragma unroll
          for (int x = 0; x < 64; ++x) m = fmaxf(m, __uint_as_float(sr[x]));
        } else {
#pragma unroll
          for (int x = 0; x < 64; ++x)
            if (x < nk) m = fmaxf(m, __uint_as_float(sr[x]));
        }
        const float mb = m * scale_log2;
        uint32_t pk[32];
        if (!masked) {
#pragma unroll
          for (int x = 0; x < 64; x += 2)
            pk[x >> 1] = tc::pack_bf16x2(
                tc::ex2_approx(fmaf(__uint_as_float(sr[x]), scale_log2, -mb)),
                tc::ex2_approx(fmaf(__uint_as_float(sr[x + 1]), scale_log2, -mb)));
        } else {
#pragma unroll
          for (int x = 0; x < 64; x += 2)
            pk[x >> 1] = tc::pack_bf16x2(
                x < nk ? tc::ex2_approx(fmaf(__uint_as_float(sr[x]), scale_log2, -mb)) : 0.f,
                x + 1 < nk ? tc::ex2_approx(fmaf(__uint_as_float(sr[x + 1]), scale_log2, -mb))
                           : 0.f);
        }
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<uint4*>(stage + tc::swz(row, c)) =
              make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        tc::fence_proxy_async();
        tc::tc_fence_before();
        tc::mbar_arrive(&sm_done[wg]);
        bad = !tc::warp_wait(&o_full[wg], u & 1);
      }
      if (!bad) {
        tc::tc_fence_after();
        // l = column d of O (the ones block)
        float linv;
        {
          uint32_t lv[16];
          tc::tmem_ld16(tmem + lane_off + Lay::kTmemO + wg * Lay::kNO + D, lv);
          tc::tmem_ld_wait();
          const float l = __uint_as_float(lv[0]);
          linv = l > 0.f ? 1.f / l : 0.f;
        }
        // O / l -> bf16, row `row` of the stage, 16-byte chunk c at slot c ^ (position & 7)
        const int key7 = (d.tile_base + row) & 7;
        uint8_t* orow = stage + row * (D * 2);
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t o[32];
          tc::tmem_ld32(tmem + lane_off + Lay::kTmemO + wg * Lay::kNO + c0, o);
          tc::tmem_ld_wait();
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            uint32_t w4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
              w4[e] = tc::pack_bf16x2(__uint_as_float(o[q4 * 8 + 2 * e]) * linv,
                                      __uint_as_float(o[q4 * 8 + 2 * e + 1]) * linv);
            const int c = (c0 >> 3) + q4;
            *reinterpret_cast<uint4*>(orow + ((c ^ key7) << 4)) =
                make_uint4(w4[0], w4[1], w4[2], w4[3]);
          }
        }
        tc::tc_fence_before();
        tc::mbar_arrive(&o_free[wg]);
        tc::fence_proxy_async();
      }
      if (tc::named_barrier_or(1 + wg, 128, bad || abort_sh != 0)) {
        ok = false;
        break;
      }
      // every row of the group is written (and fenced for the async proxy):
      // hand the stage to the store warp
      if (row == 0) {
        st_dst[st] = (int64_t)d.tile_base * (D * 2);
        st_bytes[st] = (uint32_t)d.n_valid * (D * 2);
        tc::mbar_arrive(&staged[st]);
      }
    }
    if (!ok) abort_sh = 1;
  }

  if (abort_sh && tid == 0) set_device_error(kErrTimeout);
  tc::tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) tc::tmem_dealloc(tmem, Lay::kTmemCols);
}

// out[row] = sum over valid slots of w[row, slot] * partial[inv[row * k + slot]]
// (float32, slot order); one warp per row, lane x owns elements x*E .. x*E+E-1.
template <int D>
__global__ void merge_kernel(Params P, PrefillWs ws, const int32_t* idx, const float* wts,
                             void* out, int64_t rows) {
  const int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  constexpr int E = D / 32;  // elements per lane
  const int e0 = lane * E;
  const int c = e0 >> 3, within = e0 & 7;
  // this row's slots, one per lane
  int32_t my_pos = -1;
  float my_w = 0.f;
  if (lane < P.k && idx[r * P.k + lane] >= 0) {
    my_pos = ws.inv[r * P.k + lane];
    my_w = wts[r * P.k + lane];
  }
  float acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
  for (int s = 0; s < P.k; ++s) {
    const int32_t pos = __shfl_sync(0xffffffffu, my_pos, s);
    const float w = __shfl_sync(0xffffffffu, my_w, s);
    if (pos < 0) continue;
    const uint16_t* src = reinterpret_cast<const uint16_t*>(ws.partial) + (int64_t)pos * D +
                          ((c ^ (pos & 7)) << 3) + within;
    if (E == 4) {
      const uint2 v = *reinterpret_cast<const uint2*>(src);
      acc[0] = fmaf(w, __uint_as_float(v.x << 16), acc[0]);
      acc[1] = fmaf(w, __uint_as_float(v.x & 0xFFFF0000u), acc[1]);
      acc[2] = fmaf(w, __uint_as_float(v.y << 16), acc[2]);
      acc[3] = fmaf(w, __uint_as_float(v.y & 0xFFFF0000u), acc[3]);
    } else {
      const uint32_t v = *reinterpret_cast<const uint32_t*>(src);
      acc[0] = fmaf(w, __uint_as_float(v << 16), acc[0]);
      acc[1] = fmaf(w, __uint_as_float(v & 0xFFFF0000u), acc[1]);
    }
  }
  uint16_t* o = reinterpret_cast<uint16_t*>(out) + r * D + e0;
  if (E == 4) {
    *reinterpret_cast<uint2*>(o) = make_uint2(tc::pack_bf16x2(acc[0], acc[1]),
                                              tc::pack_bf16x2(acc[2], acc[3]));
  } else {
    *reinterpret_cast<uint32_t*>(o) = tc::pack_bf16x2(acc[0], acc[1]);
  }
}

template <int D>
cudaError_t run_attn_tc(const Params& P, void* out, const int32_t* idx, const float* w,
                        const PrefillWs& ws, cudaStream_t s) {
  using Lay = AttnLayout<D>;
  cudaError_t e = set_smem(attn_tc_kernel<D>, Lay::kSmem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148, per_sm = 1;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return e;
  if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, attn_tc_kernel<D>, kThreads,
                                                         Lay::kSmem)) != cudaSuccess)
    return e;
  {
    HILS_PROFILE("prefill.attend_tc", s);
    attn_tc_kernel<D><<<sms * max(1, per_sm), kThreads, Lay::kSmem, s>>>(P, ws);
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int64_t rows = (int64_t)P.B * P.L * P.Hq;
  {
    HILS_PROFILE("prefill.merge", s);
    merge_kernel<D><<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(P, ws, idx, w, out, rows);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_tc(const Params& P, void* out, const int32_t* idx, const float* w,
                           const PrefillWs& ws, cudaStream_t s) {
  return P.d == 64 ? run_attn_tc<64>(P, out, idx, w, ws, s)
                   : run_attn_tc<128>(P, out, idx, w, ws, s);
}

}  // namespace hils
