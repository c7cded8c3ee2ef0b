// Prefill per-chunk attention (a5) and the fused, score-weighted merge (a6) on
// the 5th-generation tensor cores (tcgen05, TMEM accumulators), bf16 inputs.
//
// Work is key-major: the (row, slot) pairs are bucketed by (sequence, KV head,
// query window, chunk) and a work item is up to kItemPairs pairs of one
// bucket, so the chunk's 64 x d K and V tiles are loaded into shared memory
// once per item and shared by up to four 128-row tiles.  One persistent CTA
// per SM runs a warp-specialised pipeline over its items' tiles:
//
//   warp 0 (producer)  takes items in a fixed order.  Per tile a bulk copy of
//       its 128 pair records (query row; fusion weight with the visible keys
//       in its lowest bits) into a ring of kRing slots; per item one TMA copy of K and one of V (3-d
//       tensor map over the page pool) into one of two buffers.
//   warps 10-11 (gathers)  per tile, the pairs' query rows into one of NS
//       stages with 16-byte cp.async, 128-byte swizzled, 64 rows per warp.
//   warp 1 (MMA)  one thread issues, as each becomes ready, S = Q K^T
//       (M = 128, N = 64) into one of the two TMEM S buffers of the tile's
//       group, and O = P V (N = d) with P read from tensor memory into the
//       group's O buffer.  A stage is free once its S product is done.
//   warps 2-5, 6-9 (two softmax groups, even / odd tiles)  thread t of a
//       group owns tile row t (TMEM lane t): softmax of its 64 logits (keys
//       after the query masked in the own chunk), l = sum of the
//       probabilities, and P scaled by w / l as bf16 into the first 32
//       columns of the S buffer, so that P V is already the pair's share of
//       the output row.
//   warps 12-15 (epilogue)  tile after tile, one TMEM lane quarter each: O to
//       bf16, staged in shared memory and added into the output rows in L2
//       (red.global.add.bf16x2, 128 contiguous bytes of each of four rows per
//       warp instruction).  The output is zeroed before the kernel, and every
//       pair adds its share, so no partial results are stored.
//
// The sum over a row's k pairs is taken by bf16 atomic additions in L2, in no
// fixed order: the output is not bit-reproducible from run to run, and each
// addition rounds to bf16.
#include <cfloat>

#include "hils_common.cuh"
#include "tc_common.cuh"

namespace hils {
namespace {

constexpr int kRows = 128;        // pairs per MMA tile (M)
constexpr int kProdWarp = 0;
constexpr int kMmaWarp = 1;
constexpr int kGroupWarp0 = 2;    // group g: warps 2 + 4g .. 5 + 4g
constexpr int kGatherWarp0 = 10;  // warps 10-11: query-row gathers
constexpr int kGatherWarps = 2;
constexpr int kEpiWarp0 = 12;     // warps 12-15: epilogue, one per TMEM lane quarter
constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kRing = 8;          // tiles whose descriptors and pair records are in flight
// One ring slot of 8-byte pair records: the tile's 128, copied from the
// 16-byte boundary at or before its first, with room for the one before it
// and the rounding of the copy to 16 bytes.
constexpr uint32_t kMetaSlot = (kRows + 2) * 8;
constexpr uint32_t kStageRowBytes = 128;  // epilogue staging: 64 bf16 of one row

template <int D>
struct AttnLayout {
  static constexpr int NS = 4;                           // query stages
  static constexpr uint32_t kQBytes = kRows * D * 2;    // one query tile
  static constexpr uint32_t kKVBytes = kChunk * D * 2;  // one K (or V) tile
  static constexpr uint32_t kQ = 0;                     // NS stages
  static constexpr uint32_t kK = NS * kQBytes;          // two K buffers
  static constexpr uint32_t kV = kK + 2 * kKVBytes;     // two V buffers
  static constexpr uint32_t kStage = kV + 2 * kKVBytes; // 4 warps x 32 rows x 128 bytes
  static constexpr uint32_t kStageWarp = 32 * kStageRowBytes;
  static constexpr uint32_t kMeta = kStage + 4 * kStageWarp;   // [kRing] slots of pair records
  static constexpr uint32_t kEnd = kMeta + kRing * kMetaSlot;
  static constexpr uint32_t kSmem = kEnd + 1024;                // + slack for 1024-byte alignment
  static_assert(kSmem + 1024 <= 232448, "dynamic + static shared memory above 227 KB");
  static constexpr uint32_t kTmemCols = 512;
  // TMEM, group g at column 256 g: S buffers at +0 and +64, O (d columns) at +128
  static constexpr uint32_t kGroupCols = 256;
  static constexpr uint32_t kOCol = 128;
};

struct TileDesc {
  int32_t tile_base;  // bucket position of the tile's row 0
  int32_t n_valid;    // rows in use
  int32_t kb;         // K/V buffer
  int32_t kv_phase;   // parity of that buffer's fill
  int32_t first, last, end;
  int32_t rec0;       // record of tile row 0 in the ring slot (0 or 1)
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(Params P, PrefillWs ws, void* out, const __grid_constant__ CUtensorMap tm_kv) {
  using Lay = AttnLayout<D>;
  constexpr int NS = Lay::NS;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t q_full[NS], q_empty[NS], kv_full[2], kv_empty[2];
  __shared__ uint64_t ring_full[kRing], ring_free[kRing];
  __shared__ uint64_t s_full[2][2], sm_done[2][2], o_full[2], o_free[2], drain;
  __shared__ TileDesc desc[kRing];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~(uintptr_t)1023);
  const uint32_t sbase = tc::smem_u32(smem);
  // pair records of ring slot x, tile row r: meta[x * (kMetaSlot / 8) + desc[x].rec0 + r]
  const int2* meta = reinterpret_cast<const int2*>(smem + Lay::kMeta);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  volatile int* abort_v = &abort_sh;

  if (tid == 0) {
    for (int x = 0; x < NS; ++x) {
      tc::mbar_init(&q_full[x], 32 * kGatherWarps);   // every gather lane, once its copies landed
      tc::mbar_init(&q_empty[x], 1);  // commit of the tile's S product
    }
    for (int x = 0; x < kRing; ++x) {
      tc::mbar_init(&ring_full[x], 1);   // the producer's expect_tx arrival; the records' bytes
      tc::mbar_init(&ring_free[x], 9);   // the group's four warps, the MMA thread, the epilogue
    }
    for (int x = 0; x < 2; ++x) {
      tc::mbar_init(&kv_full[x], 1);
      tc::mbar_init(&kv_empty[x], 1);
      tc::mbar_init(&o_full[x], 1);
      tc::mbar_init(&o_free[x], 4);   // the four epilogue warps
      for (int y = 0; y < 2; ++y) {
        tc::mbar_init(&s_full[x][y], 1);
        tc::mbar_init(&sm_done[x][y], 128);
      }
    }
    tc::mbar_init(&drain, 1);
    tc::fence_mbar_init();
    abort_sh = 0;
  }
  if (warp == kMmaWarp) {
    tc::tmem_alloc(&tmem_base_sh, Lay::kTmemCols);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  const int n_items = ws.tile_off[ws.n_keys];

  if (warp == kProdWarp) {
    // --------------------------------------------------------------- producer
    // Items are taken in a fixed order (blockIdx.x, + gridDim.x, ...).  Per
    // tile: its descriptor and a bulk copy of its pair records into the next
    // ring slot; per item, first: K and V into one of the two buffers.  The
    // ring (kRing tiles) lets this run ahead of the gathers.
    const int stride = gridDim.x;
    auto item_info = [&](int it) {
      return it < n_items ? ws.items[it] : make_int4(0, 0, 0, 0);
    };
    // K/V tiles and pair records are read once: they must not push the
    // output rows (the targets of the additions) and the query rows out of L2
    const uint64_t stream_policy = tc::l2_evict_first_policy();
    int item = blockIdx.x, n_item = 0, m = 0, kv_issued = 0;
    int4 info = item_info(item), info_next = item_info(item + stride);
    bool ok = true;
    for (;; ++n_item) {
      if (__any_sync(0xffffffffu, *abort_v != 0)) {
        ok = false;
        break;
      }
      if (item >= n_items) break;
      const int4 info_after = item_info(item + 2 * stride);
      const int nt = (info.z - info.y + kRows - 1) / kRows;
      const int kb = n_item & 1;
      for (int t = 0; t < nt; ++t, ++m) {
        const int slot = m % kRing;
        if (m >= kRing && !tc::warp_wait(&ring_free[slot], ((m / kRing) - 1) & 1, wait_limit())) {
          ok = false;
          break;
        }
        if (t == 0) {
          if (n_item >= 2 && !tc::warp_wait(&kv_empty[kb], ((n_item >> 1) - 1) & 1, wait_limit())) {
            ok = false;
            break;
          }
          if (lane == 0) {
            const int key = info.x;
            const int j = key % P.max_chunks;
            const int bg = key / P.max_chunks / ws.n_win;
            const int g = bg % P.Hkv, b = bg / P.Hkv;
            int64_t page = P.block_table[(int64_t)b * P.max_chunks + j];
            if (page < 0 || page >= P.num_pages) {
              set_device_error(kErrPage);   // the tile reads page 0 instead; the call reports it
              page = 0;
            }
            const int zk = (int)((page * 2 + 0) * P.Hkv + g), zv = (int)((page * 2 + 1) * P.Hkv + g);
            tc::mbar_arrive_expect_tx(&kv_full[kb], 2 * Lay::kKVBytes);
#pragma unroll
            for (int c = 0; c < D / 64; ++c) {
              tc::tma_load_3d_hint(sbase + Lay::kK + kb * Lay::kKVBytes + c * (kChunk * 128),
                                   &tm_kv, c * 64, 0, zk, &kv_full[kb], stream_policy);
              tc::tma_load_3d_hint(sbase + Lay::kV + kb * Lay::kKVBytes + c * (kChunk * 128),
                                   &tm_kv, c * 64, 0, zv, &kv_full[kb], stream_policy);
            }
          }
          kv_issued = n_item + 1;
        }
        if (lane == 0) {
          TileDesc d{};
          d.tile_base = info.y + t * kRows;
          d.n_valid = min(kRows, info.z - d.tile_base);
          d.kb = kb;
          d.kv_phase = (n_item >> 1) & 1;
          d.first = t == 0;
          d.last = t == nt - 1;
          // the copy starts at the 16-byte boundary at or before the tile's
          // first record and covers whole 16-byte units (the workspace has
          // room after the last record)
          d.rec0 = d.tile_base & 1;
          const uint32_t bytes = ((uint32_t)(d.rec0 + d.n_valid) * 8u + 15u) & ~15u;
          desc[slot] = d;
          tc::mbar_arrive_expect_tx(&ring_full[slot], bytes);
          tc::bulk_g2s_hint(sbase + Lay::kMeta + (uint32_t)slot * kMetaSlot,
                            ws.pinfo + (d.tile_base - d.rec0), bytes, &ring_full[slot],
                            stream_policy);
        }
      }
      if (!ok) break;
      item += stride;
      info = info_next;
      info_next = info_after;
    }
    // two end markers: one for each group
    for (int e = 0; e < 2 && ok; ++e, ++m) {
      const int slot = m % kRing;
      if (m >= kRing && !tc::warp_wait(&ring_free[slot], ((m / kRing) - 1) & 1, wait_limit())) {
        ok = false;
        break;
      }
      if (lane == 0) {
        TileDesc d{};
        d.end = 1;
        desc[slot] = d;
        tc::mbar_arrive(&ring_full[slot]);
      }
    }
    if (!ok) {
      if (lane == 0) *abort_v = 1;
      // let the copies already issued land before the CTA exits (bounded waits)
      for (int x = max(0, m - kRing); x < m; ++x)
        tc::mbar_wait(&ring_full[x % kRing], (x / kRing) & 1, kDrainLimitNs);
      for (int x = max(0, kv_issued - 2); x < kv_issued; ++x)
        tc::mbar_wait(&kv_full[x & 1], (x >> 1) & 1, kDrainLimitNs);
    }
  } else if (warp >= kGatherWarp0 && warp < kEpiWarp0) {
    // ---------------------------------------------------------------- gathers
    // Tile after tile: once its records have landed and its stage is free,
    // warp w copies the query rows 64 w' .. 64 w' + 63 (w' = w - 10) into the
    // stage, 16 bytes per cp.async, in the 128-byte-swizzled K-major layout;
    // every lane arrives on the stage's barrier when its copies have landed.
    constexpr int CPR = D / 8;        // 16-byte chunks per row
    constexpr int RPI = 32 / CPR;     // rows per warp-wide copy instruction
    const int gw = warp - kGatherWarp0;
    bool ok = true;
    for (int n = 0;; ++n) {
      const int st = n % NS, slot = n % kRing;
      if (n >= NS && !tc::warp_wait(&q_empty[st], ((n / NS) - 1) & 1, wait_limit())) {
        ok = false;
        break;
      }
      if (!tc::warp_wait(&ring_full[slot], (n / kRing) & 1, wait_limit())) {
        ok = false;
        break;
      }
      const TileDesc d = desc[slot];
      if (d.end) {
        // the first end marker goes to the MMA thread through the stage barrier
        tc::mbar_arrive(&q_full[st]);
        break;
      }
      const int2* rec = meta + slot * (kMetaSlot / 8) + d.rec0;
      const uint32_t qdst = sbase + Lay::kQ + st * Lay::kQBytes;
      const uint16_t* qb = reinterpret_cast<const uint16_t*>(P.q);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int my_row = gw * 64 + h * 32 + lane;
        const int32_t my_r = my_row < d.n_valid ? rec[my_row].x : rec[0].x;
#pragma unroll
        for (int it = 0; it < 32 / RPI; ++it) {
          const int rr = it * RPI + lane / CPR, c = lane % CPR;
          const int row = gw * 64 + h * 32 + rr;
          const int32_t r = __shfl_sync(0xffffffffu, my_r, rr);
          tc::cp_async16(qdst + (uint32_t)(c >> 3) * (kRows * 128) + tc::swz(row, c & 7),
                         qb + (int64_t)r * D + c * 8, 16u);
        }
      }
      tc::cp_async_mbar_arrive(&q_full[st]);
      if (*abort_v) {
        ok = false;
        break;
      }
    }
    if (!ok) *abort_v = 1;
    tc::cp_async_wait<0>();
  } else if (warp == kMmaWarp) {
    // -------------------------------------------------------------------- MMA
    if (lane == 0) {
      constexpr uint32_t kIdS = tc::idesc_bf16(kRows, kChunk, 0);
      constexpr uint32_t kIdO = tc::idesc_bf16(kRows, D, 1);
      int ns = 0, np = 0;   // next tile to issue S for / P V for
      bool s_done = false, issued = false;
      uint64_t t_idle = 0;
      uint32_t idle = 0;
      for (;;) {
        bool progress = false;
        // O = P V of tile np once its softmax is done and the group's O is free
        if (np < ns) {
          const int g = np & 1, u = np >> 1, bf = u & 1;
          if (tc::mbar_test_wait(&sm_done[g][bf], (u >> 1) & 1) &&
              (u == 0 || tc::mbar_test_wait(&o_free[g], (u - 1) & 1))) {
            tc::tc_fence_after();
            const TileDesc d = desc[np % kRing];
            const uint32_t vb = sbase + Lay::kV + d.kb * Lay::kKVBytes;
            const uint32_t sp = tmem + g * Lay::kGroupCols + bf * kChunk;
#pragma unroll
            for (int kk = 0; kk < kChunk / 16; ++kk) {
              const uint64_t bd = tc::smem_desc(vb + kk * 2048, kChunk * 128, 1024);
              tc::mma_bf16_tmem_a(tmem + g * Lay::kGroupCols + Lay::kOCol, sp + kk * 8, bd, kIdO,
                                  kk > 0);
            }
            tc::mma_commit(&o_full[g]);
            if (d.last) tc::mma_commit(&kv_empty[d.kb]);
            tc::mbar_arrive(&ring_free[np % kRing]);
            ++np;
            progress = true;
          }
        }
        // S = Q K^T of tile ns once it is gathered and its S buffer is free:
        // the softmax of the buffer's previous tile is done and that tile's
        // P V (which reads P from the buffer) was issued before this
        if (!s_done) {
          const int st = ns % NS;
          if (tc::mbar_test_wait(&q_full[st], (ns / NS) & 1) &&
              tc::mbar_test_wait(&ring_full[ns % kRing], (ns / kRing) & 1)) {
            const TileDesc d = desc[ns % kRing];
            const int g = ns & 1, u = ns >> 1, bf = u & 1;
            if (d.end) {
              s_done = true;
            } else if ((!d.first || tc::mbar_test_wait(&kv_full[d.kb], d.kv_phase)) &&
                       (u < 2 || (np > ns - 4 &&
                                  tc::mbar_test_wait(&sm_done[g][bf], ((u >> 1) - 1) & 1)))) {
              tc::tc_fence_after();
              const uint32_t qst = sbase + Lay::kQ + st * Lay::kQBytes;
              const uint32_t kbuf = sbase + Lay::kK + d.kb * Lay::kKVBytes;
#pragma unroll
              for (int kk = 0; kk < D / 16; ++kk) {
                const uint64_t a =
                    tc::smem_desc(qst + (kk >> 2) * (kRows * 128) + (kk & 3) * 32, 16, 1024);
                const uint64_t bd =
                    tc::smem_desc(kbuf + (kk >> 2) * (kChunk * 128) + (kk & 3) * 32, 16, 1024);
                tc::mma_bf16(tmem + g * Lay::kGroupCols + bf * kChunk, a, bd, kIdS, kk > 0);
              }
              tc::mma_commit(&s_full[g][bf]);
              tc::mma_commit(&q_empty[st]);
              ++ns;
              issued = true;
              progress = true;
            }
          }
        }
        if (s_done && np == ns) break;
        if (progress) {
          idle = 0;
        } else if (*abort_v) {
          break;
        } else if ((++idle & 255u) == 0) {
          const uint64_t now = tc::globaltimer_ns();
          if (idle == 256) {
            t_idle = now;
          } else if (now - t_idle > wait_limit()) {
            *abort_v = 1;
            break;
          }
        }
      }
      // every product issued has finished before the CTA frees its TMEM
      if (issued) {
        tc::mma_commit(&drain);
        tc::mbar_wait(&drain, 0, kDrainLimitNs);
      }
    }
    __syncwarp();
  } else if (warp >= kEpiWarp0) {
    // --------------------------------------------------------------- epilogue
    // Tile after tile (both groups): O, already scaled by w / l through P, is
    // rounded to bf16 and added into the output rows.  Warp e owns TMEM lanes
    // 32 e .. 32 e + 31 (tile rows).  Each 64-column slice is staged in shared
    // memory (row r's 16-byte chunk c at chunk c ^ (r & 7)) and read back so
    // that one warp instruction adds 128 contiguous bytes into each of four
    // rows.
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    uint8_t* stg = smem + Lay::kStage + (warp - kEpiWarp0) * Lay::kStageWarp;
    uint16_t* const outp = reinterpret_cast<uint16_t*>(out);
    bool ok = true;
    for (int n = 0;; ++n) {
      const int slot = n % kRing, g = n & 1, u = n >> 1;
      if (!tc::warp_wait(&ring_full[slot], (n / kRing) & 1, wait_limit()) || *abort_v != 0) {
        ok = false;
        break;
      }
      const TileDesc d = desc[slot];
      if (d.end) break;
      const int32_t rid = row < d.n_valid ? meta[slot * (kMetaSlot / 8) + d.rec0 + row].x : -1;
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&ring_free[slot]);
      if (!tc::warp_wait(&o_full[g], u & 1, wait_limit())) {
        ok = false;
        break;
      }
      tc::tc_fence_after();
      const uint32_t to = tmem + lane_off + g * Lay::kGroupCols + Lay::kOCol;
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 64) {
        uint32_t o[64];
        {
          uint32_t a[32], b[32];
          tc::tmem_ld32(to + c0, a);
          tc::tmem_ld32(to + c0 + 32, b);
          tc::tmem_ld_wait();
#pragma unroll
          for (int x = 0; x < 32; ++x) {
            o[x] = a[x];
            o[32 + x] = b[x];
          }
        }
        if (c0 + 64 == D) {
          // all of O is in registers: the group's next P V may overwrite it
          tc::tc_fence_before();
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(&o_free[g]);
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          uint4 v;
          v.x = tc::pack_bf16x2(__uint_as_float(o[8 * q + 0]), __uint_as_float(o[8 * q + 1]));
          v.y = tc::pack_bf16x2(__uint_as_float(o[8 * q + 2]), __uint_as_float(o[8 * q + 3]));
          v.z = tc::pack_bf16x2(__uint_as_float(o[8 * q + 4]), __uint_as_float(o[8 * q + 5]));
          v.w = tc::pack_bf16x2(__uint_as_float(o[8 * q + 6]), __uint_as_float(o[8 * q + 7]));
          *reinterpret_cast<uint4*>(stg + tc::swz(lane, q)) = v;
        }
        __syncwarp();
        int32_t r[8];
        uint4 v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int src = 4 * i + (lane >> 3);
          r[i] = __shfl_sync(0xffffffffu, rid, src);
          v[i] = *reinterpret_cast<const uint4*>(stg + tc::swz(src, lane & 7));
        }
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if (r[i] >= 0) tc::red_add_bf16x8(outp + (int64_t)r[i] * D + c0 + (lane & 7) * 8, v[i]);
      }
    }
    if (!ok) *abort_v = 1;
  } else {
    // -------------------------------------------------------- softmax groups
    const int g = (warp - kGroupWarp0) >> 2;
    const int quarter = warp & 3;                   // TMEM lanes this warp may access
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t tg = tmem + lane_off + g * Lay::kGroupCols;
    const float scale_log2 = P.inv_sqrt_d * 1.4426950408889634f;
    bool ok = true;
    for (int u = 0;; ++u) {
      const int n = 2 * u + g, slot = n % kRing;
      // every wait below is on an mbarrier whose phase the whole group (or
      // the MMA thread) completes, so each warp goes its own pace; a warp
      // whose wait ran out leaves, and the others follow once theirs do
      if (!tc::warp_wait(&ring_full[slot], (n / kRing) & 1, wait_limit()) || *abort_v != 0) {
        ok = false;
        break;
      }
      const TileDesc d = desc[slot];
      if (d.end) break;
      const bool row_valid = row < d.n_valid;
      const int2 rec = meta[slot * (kMetaSlot / 8) + d.rec0 + row];
      const int nk = row_valid ? (rec.y & 63) + 1 : kChunk;
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&ring_free[slot]);
      const int bf = u & 1;
      if (!tc::warp_wait(&s_full[g][bf], (u >> 1) & 1, wait_limit())) {
        ok = false;
        break;
      }
      tc::tc_fence_after();
      uint32_t sr[64];
      {
        uint32_t a[32], c[32];
        tc::tmem_ld32(tg + bf * kChunk, a);
        tc::tmem_ld32(tg + bf * kChunk + 32, c);
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
      float l4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int x = 0; x < 64; ++x) {
        float e = tc::ex2_approx(fmaf(__uint_as_float(sr[x]), scale_log2, -mb));
        if (masked) e = x < nk ? e : 0.f;
        l4[x & 3] += e;
        sr[x] = __float_as_uint(e);
      }
      const float l = (l4[0] + l4[1]) + (l4[2] + l4[3]);
      // P scaled by the fusion weight over l, so that P V is already this
      // pair's share of the output
      const float scale = (row_valid && l > 0.f) ? __int_as_float(rec.y & ~63) / l : 0.f;
      uint32_t pk[32];
#pragma unroll
      for (int x = 0; x < 32; ++x)
        pk[x] = tc::pack_bf16x2(__uint_as_float(sr[2 * x]) * scale,
                                __uint_as_float(sr[2 * x + 1]) * scale);
      // P over the first 32 columns of the S buffer (the logits are in registers)
      tc::tmem_st32(tg + bf * kChunk, pk);
      tc::tmem_st_wait();
      tc::tc_fence_before();
      tc::mbar_arrive(&sm_done[g][bf]);
    }
    if (!ok) *abort_v = 1;
  }

  if (*abort_v && tid == 0) set_device_error(kErrTimeout);
  tc::tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) tc::tmem_dealloc(tmem, Lay::kTmemCols);
}

template <int D>
cudaError_t run_attn_tc(const Params& P, void* out, const PrefillWs& ws, cudaStream_t s) {
  using Lay = AttnLayout<D>;
  const int64_t rows = (int64_t)P.B * P.L * P.Hq;
  CUtensorMap tm_kv;
  {
    // pages [num_pages][2][Hkv][64][D] as (D, 64 slots, page * 2 * Hkv + kind * Hkv + head)
    const uint64_t dims[3] = {(uint64_t)D, (uint64_t)kChunk, (uint64_t)P.num_pages * 2 * P.Hkv};
    const uint64_t strides[2] = {(uint64_t)D * 2, (uint64_t)kChunk * D * 2};
    const uint32_t box[3] = {64, (uint32_t)kChunk, 1};
    cudaError_t e = encode_tmap_bf16(&tm_kv, 3, P.pages, dims, strides, box);
    if (e != cudaSuccess) return e;
  }
  if (P.num_pages * 2 * P.Hkv >= ((int64_t)1 << 31)) return cudaErrorInvalidValue;
  cudaError_t e = set_smem(attn_tc_kernel<D>, Lay::kSmem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return e;
  // every pair adds its share into the output
  if ((e = cudaMemsetAsync(out, 0, (size_t)rows * D * 2, s)) != cudaSuccess) return e;
  {
    HILS_PROFILE("prefill.attend_tc", s);
    attn_tc_kernel<D><<<sms, kThreads, Lay::kSmem, s>>>(P, ws, out, tm_kv);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_tc(const Params& P, void* out, const PrefillWs& ws, cudaStream_t s) {
  return P.d == 64 ? run_attn_tc<64>(P, out, ws, s) : run_attn_tc<128>(P, out, ws, s);
}

}  // namespace hils
