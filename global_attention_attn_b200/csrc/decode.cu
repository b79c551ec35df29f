// Decode and speculative verification: q_len query tokens per sequence (1 for a decode
// step, 2..8 draft tokens to verify) over the ring (sliding-window layers) or paged
// (global layers) KV cache, split-KV with a combine pass.
//
// Decode streams the cache once: it is HBM-bound (16 FLOP per byte for the global layer,
// 8 for the sliding layer), so the contractions run on mma.sync m16n8k16 with the query
// heads of one KV group (GQA, "Model techniques map" page, "Grouped-query attention": 16
// query heads per KV head on global layers, 8 on sliding layers) times the draft tokens as
// the M rows.  Row r of a unit's rows is draft r / G, head r % G: a block of 16 rows is one
// draft's 16 heads (global layers) or two drafts' 8 heads (sliding layers; one real draft
// and 8 padding rows when decoding).  The sink logit ("Learnable attention sink") joins
// the final denominator only.  Each draft row has its own position (ctx - q_len + i), so
// its own rotary angle and its own causal (and window) limit: draft i sees the context and
// drafts 0..i, as the draft tokens of the speculative decoding the serving pages run
// (vLLM recipe page, DFlash; SGLang cookbook page; miles docs section 4.2, EAGLE with 4
// draft tokens) must be scored.
//
// Work unit = (split, sequence, KV head, row part).  A CTA holds groups of one producer
// warp and NC consumer warps:
//   producer warp: reads the context length and page ids of the next unit, computes the
//     unit's rotary cos / sin rows (float64 angles, one row per draft), TMA-loads the
//     unit's query rows (NC blocks of 16) into a double-buffered tile, then streams the
//     unit's keys and values as 16-key TMA tiles (128-byte swizzle) through a ring of
//     stages that all NC consumers read;
//   consumer warp c: takes row block (row part * NC + c), builds its query fragments from
//     shared memory with ldmatrix, rotates dims 0..63 in registers, then runs QK^T, the
//     online softmax and PV over the tiles with mma.sync, and writes its rows' result (the
//     final output when a sequence has one split, else partials).
// A ring cache is read in slot order with each slot's position recovered from the context
// length: attention does not depend on key order.
#include <cuda_bf16.h>

#include "common.cuh"
#include "ptx.cuh"
#include "../../include/mimoattn.h"

namespace mimo {

namespace {

constexpr int kTileK = 16;                     // keys per TMA tile
constexpr int kQChunk = 16 * 128;              // 16 rows x 64 dims x 2 bytes
constexpr int kQBlock = 3 * kQChunk;           // one 16-row block of queries, 192 dims
constexpr int kMaxDrafts = 8;
constexpr int kMaxTable = 1024;                // sequences of the ordered split enumeration

// Shared memory of one CTA.  A stage holds one 16-key tile: K as three 64-element
// chunks, V as two; bf16 rows are 128 bytes (128-byte swizzle), E4M3 rows 64 bytes
// (64-byte swizzle, twice the stages for the same bytes in flight).
// Groups per CTA and stages per group: at most 8 warps per CTA, so that a consumer keeps
// its query fragments and output accumulators in registers (255 per thread), and 40..80 KB
// of keys and values in flight per group.
template <bool FP8, int NC>
struct DecodeLayout {
  static constexpr int kGroups = NC == 1 ? 4 : (NC == 2 ? 2 : 1);  // producer + NC consumers each
  static constexpr int kThreads = kGroups * (1 + NC) * 32;
  static constexpr int kRowBytes = FP8 ? 64 : 128;
  static constexpr int kChunk = kTileK * kRowBytes;
  static constexpr int kStageBytes = 5 * kChunk;
  static constexpr int kStages = (FP8 ? 2 : 1) * (NC == 1 ? 4 : (NC == 2 ? 6 : 8));
  static constexpr int kGroupBytes = kStages * kStageBytes + 2 * NC * kQBlock;
  // unit fields + one (cos, sin) row of 32 frequencies per draft
  static constexpr int kInfoBytes = 64 + (NC == 1 ? 1 : kMaxDrafts) * 32 * 8;
  static constexpr int kOffInfo = kGroups * kGroupBytes;
  static constexpr int kOffBar = kOffInfo + kGroups * 2 * kInfoBytes;
  static constexpr int kBarsPerGroup = 2 * kStages + 4;  // full, empty, q_full[2], q_empty[2]
  static constexpr int kOffTbl = kOffBar + kGroups * kBarsPerGroup * 8 + 16;
  static constexpr int kSmemBytes = kOffTbl + 2 * (kMaxTable + 1) * 4 + 1024;
  static_assert(kGroupBytes % 1024 == 0 && kStageBytes % 1024 == 0 && kQBlock % 1024 == 0, "swizzle alignment");
  static_assert(kInfoBytes % 16 == 0 && kOffBar % 8 == 0, "info / barrier alignment");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void mma_bf16(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// fp16 operands: the rotated dims 0..63 (fp16 in the query fragments and in the caches)
__device__ __forceinline__ void mma_f16(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Unit fields the producer hands to its consumers with the query tile.
struct UnitInfo {
  int s, g, split, ctx, k_begin, k_end, t0, nt;  // nt < 0: no more units
  int rp, pad[7];
};
static_assert(sizeof(UnitInfo) == 64, "unit fields");

// First key position of a sequence's unit range: the earliest window start of its q_len
// query rows (row i at position ctx - q_len + i), or 0 for global attention.
__device__ __forceinline__ int unit_lo(const DecodeParams& p, int ctx) {
  return p.window > 0 ? max(0, ctx - p.q_len + 1 - p.window) : 0;
}

// Work unit u of the dense space [split][sequence][kv head][row part]; false if it has no keys.
__device__ __forceinline__ bool unit_at(const DecodeParams& p, int u, UnitInfo& U) {
  const int per_split = p.batch * p.hkv * p.n_rp;
  U.split = u / per_split;
  int rem = u - U.split * per_split;
  U.s = rem / (p.hkv * p.n_rp);
  rem -= U.s * (p.hkv * p.n_rp);
  U.g = rem / p.n_rp;
  U.rp = rem - U.g * p.n_rp;
  U.ctx = p.seq_lens[U.s];
  if (U.ctx < p.q_len) return false;
  U.k_begin = unit_lo(p, U.ctx) + U.split * p.split_len;
  if (U.k_begin >= U.ctx) return false;
  U.k_end = min(U.k_begin + p.split_len, U.ctx);
  if (p.cache_kind == MIMO_CACHE_RING) {
    U.t0 = 0;
    U.nt = p.ring_slots / kTileK;  // every slot of the ring, in slot order
  } else {
    U.t0 = U.k_begin / kTileK;
    U.nt = (U.k_end - 1) / kTileK - U.t0 + 1;
  }
  return true;
}

// Keys of sequence s the unit range covers.
__device__ __forceinline__ int seq_keys(const DecodeParams& p, int ctx) {
  if (ctx < p.q_len) return 0;
  return ctx - unit_lo(p, ctx);
}

// Largest s in [0, n) with tbl[s] <= x, for a prefix table with tbl[0] = 0 <= x < tbl[n].
__device__ __forceinline__ int find_seq(const int* tbl, int n, int x) {
  int lo = 0, hi = n;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (tbl[mid] <= x) lo = mid;
    else hi = mid;
  }
  return lo;
}

// Unit v of the ordered enumeration: first every full split (split_len keys) of every
// sequence, then the shorter last splits, so that a round-robin deal over the groups gives
// each group the same number of full units.  tbl_full / tbl_part are prefix sums over
// sequences of the full-split count and of "has a shorter last split".  The row parts of a
// (split, sequence, KV head) are consecutive units: their groups read the same tiles at about
// the same time, so the second read comes from L2.
__device__ __forceinline__ void unit_ordered(const DecodeParams& p, const int* tbl_full, const int* tbl_part, int v,
                                             UnitInfo& U) {
  int x = v / (p.hkv * p.n_rp);
  const int rem = v - x * (p.hkv * p.n_rp);
  U.g = rem / p.n_rp;
  U.rp = rem - U.g * p.n_rp;
  const int F = tbl_full[p.batch];
  if (x < F) {
    U.s = find_seq(tbl_full, p.batch, x);
    U.split = x - tbl_full[U.s];
  } else {
    x -= F;
    U.s = find_seq(tbl_part, p.batch, x);
    U.split = tbl_full[U.s + 1] - tbl_full[U.s];
  }
  U.ctx = p.seq_lens[U.s];
  U.k_begin = unit_lo(p, U.ctx) + U.split * p.split_len;
  U.k_end = min(U.k_begin + p.split_len, U.ctx);
  U.t0 = U.k_begin / kTileK;
  U.nt = (U.k_end - 1) / kTileK - U.t0 + 1;
}

}  // namespace

template <bool FP8, int NC>
__global__ void __launch_bounds__(DecodeLayout<FP8, NC>::kThreads, 1)
    decode_kernel(const __grid_constant__ DecodeParams p) {
  using Ly = DecodeLayout<FP8, NC>;
  constexpr int kGroups = Ly::kGroups;
  constexpr int kStages = Ly::kStages, kStageBytes = Ly::kStageBytes, kChunk = Ly::kChunk;
  constexpr int kGroupBytes = Ly::kGroupBytes, kOffInfo = Ly::kOffInfo, kOffBar = Ly::kOffBar;
  constexpr int kInfoBytes = Ly::kInfoBytes, kBarsPerGroup = Ly::kBarsPerGroup, kOffTbl = Ly::kOffTbl;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool producer = warp < kGroups;
  const int grp = producer ? warp : (warp - kGroups) / NC;
  const int cix = producer ? 0 : (warp - kGroups) % NC;  // consumer index within the group
  const uint32_t region = sbase + grp * kGroupBytes;      // stages, then the two query tiles
  const uint32_t qtile0 = region + kStages * kStageBytes;
  uint8_t* info = smem + kOffInfo + grp * 2 * kInfoBytes;
  auto info_at = [&](int b) { return reinterpret_cast<UnitInfo*>(info + b * kInfoBytes); };
  const uint32_t bar0 = sbase + kOffBar + grp * kBarsPerGroup * 8;
  auto full = [&](int i) { return bar0 + 8 * i; };
  auto empty = [&](int i) { return bar0 + 8 * (kStages + i); };
  auto q_full = [&](int b) { return bar0 + 8 * (2 * kStages + b); };
  auto q_empty = [&](int b) { return bar0 + 8 * (2 * kStages + 2 + b); };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffBar + kGroups * kBarsPerGroup * 8);
  unsigned* status = p.status;
  if (producer && lane == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(full(i), 1);
      mbar_init(empty(i), NC);  // every consumer of the group reads every stage
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(q_full(b), 2);  // the query copies' byte count, and the unit fields written
      mbar_init(q_empty(b), NC);
    }
    if (grp == 0) *abort_flag = 0;
    fence_mbar_init();
  }
  // split-KV with few enough sequences: enumerate only the units that have keys, full splits first
  const bool ordered = p.max_splits > 1 && p.batch <= kMaxTable && p.cache_kind == MIMO_CACHE_PAGED;
  int* tbl_full = reinterpret_cast<int*>(smem + kOffTbl);
  int* tbl_part = tbl_full + kMaxTable + 1;
  if (ordered && warp == kGroups) {
    int carry_f = 0, carry_p = 0;
    if (lane == 0) tbl_full[0] = tbl_part[0] = 0;
    for (int base = 0; base < p.batch; base += 32) {
      const int s = base + lane;
      int keys = s < p.batch ? seq_keys(p, p.seq_lens[s]) : 0;
      if (keys > p.max_splits * p.split_len) {  // a context beyond max_seq_len
        atomicOr(status, MIMO_STATUS_BAD_INDEX);
        keys = p.max_splits * p.split_len;
      }
      int f = keys / p.split_len, q = keys % p.split_len ? 1 : 0;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int uf = __shfl_up_sync(0xffffffffu, f, d), uq = __shfl_up_sync(0xffffffffu, q, d);
        if (lane >= d) {
          f += uf;
          q += uq;
        }
      }
      if (s < p.batch) {
        tbl_full[s + 1] = carry_f + f;
        tbl_part[s + 1] = carry_p + q;
      }
      carry_f += __shfl_sync(0xffffffffu, f, 31);
      carry_p += __shfl_sync(0xffffffffu, q, 31);
    }
  }
  __syncthreads();
  const int n_units = ordered ? (tbl_full[p.batch] + tbl_part[p.batch]) * p.hkv * p.n_rp
                              : p.batch * p.hkv * p.n_rp * p.max_splits;
  const int wg = blockIdx.x * kGroups + grp;
  const int n_grp = gridDim.x * kGroups;
  auto wait_w = [&](uint32_t bar, uint32_t parity) -> bool {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, status, MIMO_STATUS_TIMEOUT));
  };
  const int G = p.group;
  const int rows_per_block = 16 / G;  // query rows (drafts) per 16-row block: 1 (G = 16) or 2 (G = 8)

  if (producer) {
    // ------------------------------------------------------------ producer warp
    if (lane == 0) {
      tma_prefetch(&p.tm_q);
      tma_prefetch(&p.tm_k);
      tma_prefetch(&p.tm_v);
    }
    int it = 0, n = 0;
    bool ok = true;
    const bool ring = p.cache_kind == MIMO_CACHE_RING;
    for (int u = wg; u < n_units && ok; u += n_grp) {
      UnitInfo U;
      int row_l = 0, p0 = 0;
      if (ring) {
        // A ring unit's copies do not depend on the context length (the whole ring, the
        // sequence's query rows): they are issued before it is read, and its latency, the
        // rotary rows and the unit fields overlap them.  A sequence shorter than q_len
        // (invalid) is still read and reported.
        U.split = 0;
        U.s = u / (p.hkv * p.n_rp);
        const int rem = u - U.s * (p.hkv * p.n_rp);
        U.g = rem / p.n_rp;
        U.rp = rem - U.g * p.n_rp;
        U.t0 = 0;
        U.nt = p.ring_slots / kTileK;  // every slot of the ring, in slot order
      } else {
        if (ordered) unit_ordered(p, tbl_full, tbl_part, u, U);
        else if (!unit_at(p, u, U)) continue;
        // cache row of page i of the unit in lane i (a unit spans at most 32 pages)
        p0 = U.k_begin / kPage;
        if (lane <= (U.k_end - 1) / kPage - p0) {
          const int pi = p0 + lane;
          int page = pi < p.max_pages ? p.block_table[long(U.s) * p.max_pages + pi] : -1;
          if (page < 0 || page >= p.num_pages) {
            atomicOr(status, MIMO_STATUS_BAD_INDEX);
            page = 0;
          }
          row_l = page * kPage;
        }
      }
      // the query blocks of the unit's row part
      const int b = n & 1;
      if (n >= 2 && !(ok = wait_w(q_empty(b), ((n >> 1) - 1) & 1))) break;
      if (lane == 0) {
        const int blk0 = U.rp * NC;
        const int nblk = min(NC, p.n_blocks - blk0);
        const uint32_t dst = qtile0 + b * NC * kQBlock;
        mbar_expect_tx(q_full(b), nblk * kQBlock);
        const int h0 = U.g * G;
        for (int c = 0; c < nblk; ++c) {
          const int qrow = U.s * p.q_len + (blk0 + c) * rows_per_block;
          tma_load_3d(dst + c * kQBlock, &p.tm_q, q_full(b), 0, h0, qrow);
          tma_load_3d(dst + c * kQBlock + kQChunk, &p.tm_q, q_full(b), 64, h0, qrow);
          tma_load_3d(dst + c * kQBlock + 2 * kQChunk, &p.tm_q, q_full(b), 128, h0, qrow);
        }
      }
      ++n;
      // the unit's fields and rotary rows go out with the second arrival on q_full: for a
      // ring after the first stages' copies are on their way, else at once
      const int first = ring ? min(U.nt, kStages) : 0;
      auto publish = [&]() {
        if (ring) {
          U.ctx = p.seq_lens[U.s];
          if (U.ctx < p.q_len && lane == 0) atomicOr(status, MIMO_STATUS_BAD_INDEX);
          U.k_begin = unit_lo(p, U.ctx);
          U.k_end = U.ctx;
        }
        UnitInfo* I = info_at(b);
        float2* csr = reinterpret_cast<float2*>(I + 1);
        // one row per draft of the unit's blocks, padding drafts included (finite angles for
        // the rows that only fill a block)
        const int n_cs = NC == 1 ? 1 : p.n_blocks * rows_per_block;
        for (int i = 0; i < n_cs; ++i) {
          float c, s;
          rope_cos_sin(U.ctx - p.q_len + i, p.rope.inv_freq[lane], &c, &s);
          csr[i * 32 + lane] = make_float2(c, s);
        }
        if (lane == 0) *I = U;
        __syncwarp();
        if (lane == 0) mbar_arrive(q_full(b));
      };
      if (first == 0) publish();
      for (int t = 0; t < U.nt; ++t, ++it) {
        int row;
        if (ring) {
          row = U.s * p.ring_slots + kTileK * t;
        } else {
          const int key = (U.t0 + t) * kTileK;
          row = __shfl_sync(0xffffffffu, row_l, key / kPage - p0) + key % kPage;
        }
        const int st = it % kStages;
        if (it >= kStages && !(ok = wait_w(empty(st), ((it / kStages) - 1) & 1))) break;
        if (lane == 0) {
          const uint32_t dst = region + st * kStageBytes;
          mbar_expect_tx(full(st), kStageBytes);
          tma_load_3d(dst, &p.tm_k, full(st), 0, U.g, row);
          tma_load_3d(dst + kChunk, &p.tm_k, full(st), 64, U.g, row);
          tma_load_3d(dst + 2 * kChunk, &p.tm_k, full(st), 128, U.g, row);
          tma_load_3d(dst + 3 * kChunk, &p.tm_v, full(st), 0, U.g, row);
          tma_load_3d(dst + 4 * kChunk, &p.tm_v, full(st), 64, U.g, row);
        }
        __syncwarp();
        if (t + 1 == first) publish();
      }
      if (!ok) break;
    }
    if (ok) {
      // end of the unit stream
      const int b = n & 1;
      if (n < 2 || (ok = wait_w(q_empty(b), ((n >> 1) - 1) & 1))) {
        if (lane == 0) {
          info_at(b)->nt = -1;
          mbar_arrive(q_full(b));  // both arrivals: no copy goes with the end marker
          mbar_arrive(q_full(b));
        }
      }
    }
    if (!ok && lane == 0) {
      // let the copies already issued land before the CTA leaves
      int dummy = 0;
      for (int k = it - kStages < 0 ? 0 : it - kStages; k < it; ++k)
        mbar_wait(full(k % kStages), (k / kStages) & 1, &dummy, nullptr, 0, 50000000ull);
      for (int k = n - 2 < 0 ? 0 : n - 2; k < n; ++k)
        mbar_wait(q_full(k & 1), (k >> 1) & 1, &dummy, nullptr, 0, 50000000ull);
    }
    return;
  }

  // ------------------------------------------------------------ consumer warp
  const int q4 = lane & 3, r0 = lane >> 2, r1 = r0 + 8;
  int it = 0;
  for (int n = 0;; ++n) {
    const int b = n & 1;
    if (!wait_w(q_full(b), (n >> 1) & 1)) return;
    const UnitInfo* I = info_at(b);
    const int nt = I->nt;
    if (nt < 0) return;
    const int s = I->s, g = I->g, split = I->split, ctx = I->ctx, k_begin = I->k_begin, k_end = I->k_end,
              t0 = I->t0;
    const int blk = I->rp * NC + cix;     // this consumer's 16-row block of the unit
    const bool active = blk < p.n_blocks;  // a row part's last consumers may have no block
    // rows r0 / r1 of the block: draft and query position, and the visible key range
    int draft[2], lo_r[2], hi_r[2];
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int rr = blk * 16 + (half ? r1 : r0);
      draft[half] = rr / G;
      const int pos = ctx - p.q_len + draft[half];
      const bool valid = active && draft[half] < p.q_len;
      lo_r[half] = valid ? (p.window > 0 ? max(k_begin, pos - p.window + 1) : k_begin) : 1;
      hi_r[half] = valid ? min(k_end - 1, pos) : 0;
    }
    // ---- query fragments (A of m16n8k16) from the swizzled block
    uint32_t qa[12][4];
    float q_amax = 0.f;  // largest rotated (or, for E4M3, converted) query component
    const float2* csr = reinterpret_cast<const float2*>(I + 1);
    // (cos, sin) pairs of frequencies j, j + 1 for the row of fragment element e (even e: row
    // r0, odd e: row r1)
    auto cs_pair = [&](int e, int j) {
      const float2* c = csr + (NC == 1 ? 0 : draft[e & 1] * 32) + j;
      return make_float4(c[0].x, c[0].y, c[1].x, c[1].y);
    };
    const uint32_t qt = qtile0 + b * NC * kQBlock + cix * kQBlock;
    if (active) {
      if constexpr (!FP8) {
        const int row = (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
        for (int kk = 0; kk < 12; ++kk) {
          const int unit16 = ((kk & 3) * 2 + (lane >> 4)) ^ (row & 7);
          ldsm_x4(qt + (kk >> 2) * kQChunk + row * 128 + unit16 * 16, qa[kk]);
        }
        // dims j < 32 (k-steps 0, 1) pair with dims j + 32 (k-steps 2, 3) in the same register slot
#pragma unroll
        for (int kk = 0; kk < 2; ++kk)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int j0 = 16 * kk + 2 * q4 + ((e & 2) ? 8 : 0);
            const float4 t = cs_pair(e, j0);  // (cos, sin) of frequencies j0, j0 + 1
            const uint32_t xw = qa[kk][e], yw = qa[kk + 2][e];
            const float x0 = lo_bf16(xw), x1 = hi_bf16(xw), y0 = lo_bf16(yw), y1 = hi_bf16(yw);
            qa[kk][e] = pack2_f16_sat(x0 * t.x - y0 * t.y, x1 * t.z - y1 * t.w, q_amax);
            qa[kk + 2][e] = pack2_f16_sat(y0 * t.x + x0 * t.y, y1 * t.z + x1 * t.w, q_amax);
          }
      } else {
        // E4M3 keys are read with ldmatrix as pairs of bytes, which gives thread (r0, q4) the
        // 4 consecutive dims 4q4..4q4+3 of a 16-dim step: the step's k order is permuted the
        // same way here (k 2q4, 2q4+1 <- dims 4q4, 4q4+1; k 2q4+8, 2q4+9 <- dims 4q4+2, 4q4+3),
        // which leaves the dot products unchanged.  Everything runs in fp16.
#pragma unroll
        for (int kk = 0; kk < 12; ++kk) {
          const int unit16 = 2 * (kk & 3) + (q4 >> 1);
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            const int row = hf ? r1 : r0;
            const uint2 w = *reinterpret_cast<const uint2*>(smem + (qt - sbase) + (kk >> 2) * kQChunk + row * 128 +
                                                            ((unit16 ^ (row & 7)) << 4) + 8 * (q4 & 1));
            qa[kk][hf] = w.x;      // dims 4q4, 4q4 + 1 of the step
            qa[kk][2 + hf] = w.y;  // dims 4q4 + 2, 4q4 + 3
          }
        }
#pragma unroll
        for (int kk = 0; kk < 2; ++kk)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int j0 = 16 * kk + 4 * q4 + ((e & 2) ? 2 : 0);
            const float4 t = cs_pair(e, j0);
            const uint32_t xw = qa[kk][e], yw = qa[kk + 2][e];
            const float x0 = lo_bf16(xw), x1 = hi_bf16(xw), y0 = lo_bf16(yw), y1 = hi_bf16(yw);
            qa[kk][e] = pack2_f16_sat(x0 * t.x - y0 * t.y, x1 * t.z - y1 * t.w, q_amax);
            qa[kk + 2][e] = pack2_f16_sat(y0 * t.x + x0 * t.y, y1 * t.z + x1 * t.w, q_amax);
          }
#pragma unroll
        for (int kk = 4; kk < 12; ++kk)
#pragma unroll
          for (int e = 0; e < 4; ++e) qa[kk][e] = pack2_f16_sat(lo_bf16(qa[kk][e]), hi_bf16(qa[kk][e]), q_amax);
      }
    }
    // padding rows (past the draft count, or beyond the batch) hold other queries or zeros:
    // report a range overflow only where the block has a valid row
    if (q_amax > kF16Max && (hi_r[0] >= lo_r[0] || hi_r[1] >= lo_r[1])) atomicOr(status, MIMO_STATUS_RANGE);
    __syncwarp();
    if (lane == 0) mbar_arrive(q_empty(b));
    const float c_log2 = FP8 ? p.scale_log2 * p.k_dequant[g] : p.scale_log2;
    const float v_deq = FP8 ? p.v_dequant[g] : 1.f;

    // ring: the slot of position kp is kp mod R, and the ring holds positions ctx-R .. ctx-1,
    // so slot j holds position ctx - R + ((j + ring_off) mod R) with ring_off = (R - ctx) mod R
    const int R = p.ring_slots;
    const int ring_off = p.cache_kind == MIMO_CACHE_RING ? ((R - ctx) % R + R) % R : 0;
    // a paged tile whose keys every row of the block sees needs no mask: [lo_all, hi_all] is the
    // key range all of the block's rows see (empty when a row is padding)
    const int lo_all = __reduce_max_sync(0xffffffffu, max(lo_r[0], lo_r[1]));
    const int hi_all = __reduce_min_sync(0xffffffffu, min(hi_r[0], hi_r[1]));
    float m_r[2] = {-INFINITY, -INFINITY};
    float l_r[2] = {0.f, 0.f};
    float o[16][4];
#pragma unroll
    for (int i = 0; i < 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;

    for (int t = 0; t < nt; ++t, ++it) {
      const int st = it % kStages;
      if (!wait_w(full(st), (it / kStages) & 1)) return;
      if (!active) {  // a block past the unit's rows: only the stage's release
        __syncwarp();
        if (lane == 0) mbar_arrive(empty(st));
        continue;
      }
      const uint32_t kb = region + st * kStageBytes;
      const uint32_t vb = kb + 3 * kChunk;
      // two accumulators per key half (even / odd k-steps) halve the dependent MMA chain
      float acc[4][4];
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
      if constexpr (!FP8) {
        // B fragments of K^T: matrices (keys 0-7 | 8-15) x (dims lo 8 | hi 8);
        // rows are 128-byte swizzled (16-byte unit u of row k sits at u ^ (k & 7))
        const int key = (lane & 7) + (lane >> 4) * 8;
        const int dhalf = (lane >> 3) & 1;
#pragma unroll
        for (int kk = 0; kk < 12; ++kk) {
          const int unit16 = ((kk & 3) * 2 + dhalf) ^ (key & 7);
          uint32_t bf[4];
          ldsm_x4(kb + (kk >> 2) * kChunk + key * 128 + unit16 * 16, bf);
          float* a0 = acc[kk & 1];
          float* a1 = acc[2 + (kk & 1)];
          if (kk < 4) {
            mma_f16(a0, qa[kk], bf[0], bf[1]);
            mma_f16(a1, qa[kk], bf[2], bf[3]);
          } else {
            mma_bf16(a0, qa[kk], bf[0], bf[1]);
            mma_bf16(a1, qa[kk], bf[2], bf[3]);
          }
        }
      } else {
        // matrices (keys 0-7 | 8-15) x (dims 0-15 | 16-31) of a 32-dim group, 64-byte rows
        // swizzled by the 64-byte pattern (16-byte unit u of row k sits at u ^ ((k >> 1) & 3))
        const int key = (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
        for (int g32 = 0; g32 < 6; ++g32) {
          const int unit16 = 2 * (g32 & 1) + (lane >> 4);
          uint32_t bf[4];
          ldsm_x4(kb + (g32 >> 1) * kChunk + key * 64 + ((unit16 ^ ((key >> 1) & 3)) << 4), bf);
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            const int kk = 2 * g32 + hf;
            const uint32_t m_lo = bf[2 * hf], m_hi = bf[2 * hf + 1];  // keys 0-7, keys 8-15
            mma_f16(acc[kk & 1], qa[kk], f16x2_from_e4m3x2(uint16_t(m_lo)), f16x2_from_e4m3x2(uint16_t(m_lo >> 16)));
            mma_f16(acc[2 + (kk & 1)], qa[kk], f16x2_from_e4m3x2(uint16_t(m_hi)),
                    f16x2_from_e4m3x2(uint16_t(m_hi >> 16)));
          }
        }
      }
      float s0[4], s1[4];  // keys 2q4, 2q4+1 (rows r0, r0, r1, r1) and the same + 8
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        s0[i] = acc[0][i] + acc[1][i];
        s1[i] = acc[2][i] + acc[3][i];
      }
      // positions of this thread's four key columns, visible or not to each of its two rows
      const bool interior = p.cache_kind == MIMO_CACHE_PAGED && (t0 + t) * kTileK >= lo_all &&
                            (t0 + t) * kTileK + kTileK - 1 <= hi_all;
#pragma unroll
      for (int e = 0; e < 4 && !interior; ++e) {
        const int col = ((e & 2) ? 8 : 0) + 2 * q4 + (e & 1);  // within the 16-key tile
        int kp;
        if (p.cache_kind == MIMO_CACHE_RING) {
          const int j = kTileK * t + col + ring_off;  // < 2 R
          kp = ctx - R + (j >= R ? j - R : j);
        } else {
          kp = (t0 + t) * kTileK + col;
        }
        float* sv = (e & 2) ? s1 : s0;  // column e: sv[e & 1] for row r0, sv[2 + (e & 1)] for row r1
        if (!(kp >= lo_r[0] && kp <= hi_r[0])) sv[e & 1] = -INFINITY;
        if (!(kp >= lo_r[1] && kp <= hi_r[1])) sv[2 + (e & 1)] = -INFINITY;
      }
      float mx0 = fmaxf(fmaxf(s0[0], s0[1]), fmaxf(s1[0], s1[1]));
      float mx1 = fmaxf(fmaxf(s0[2], s0[3]), fmaxf(s1[2], s1[3]));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
      const float mn0 = fmaxf(m_r[0], mx0 * c_log2), mn1 = fmaxf(m_r[1], mx1 * c_log2);
      // a tile may be fully masked (split edges, padding rows): reference 0 then
      const float mu0 = mn0 == -INFINITY ? 0.f : mn0, mu1 = mn1 == -INFINITY ? 0.f : mn1;
      const float al0 = ex2(m_r[0] - mu0), al1 = ex2(m_r[1] - mu1);
      m_r[0] = mn0;
      m_r[1] = mn1;
      float p0[4], p1[4];
      p0[0] = ex2(fmaf(s0[0], c_log2, -mu0));
      p0[1] = ex2(fmaf(s0[1], c_log2, -mu0));
      p0[2] = ex2(fmaf(s0[2], c_log2, -mu1));
      p0[3] = ex2(fmaf(s0[3], c_log2, -mu1));
      p1[0] = ex2(fmaf(s1[0], c_log2, -mu0));
      p1[1] = ex2(fmaf(s1[1], c_log2, -mu0));
      p1[2] = ex2(fmaf(s1[2], c_log2, -mu1));
      p1[3] = ex2(fmaf(s1[3], c_log2, -mu1));
      l_r[0] = l_r[0] * al0 + p0[0] + p0[1] + p1[0] + p1[1];
      l_r[1] = l_r[1] * al1 + p0[2] + p0[3] + p1[2] + p1[3];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        o[i][0] *= al0;
        o[i][1] *= al0;
        o[i][2] *= al1;
        o[i][3] *= al1;
      }
      uint32_t pa[4];
      if constexpr (!FP8) {
        pa[0] = pack2_bf16(p0[0], p0[1]);
        pa[1] = pack2_bf16(p0[2], p0[3]);
        pa[2] = pack2_bf16(p1[0], p1[1]);
        pa[3] = pack2_bf16(p1[2], p1[3]);
        // B fragments of V (trans): matrices (keys 0-7 | 8-15) x (dims d0 .. d0+7 | d0+8 ..)
        const int key = (lane & 7) + ((lane >> 3) & 1) * 8;
        const int dq = lane >> 4;
#pragma unroll
        for (int n2 = 0; n2 < 8; ++n2) {
          const int unit16 = ((n2 & 3) * 2 + dq) ^ (key & 7);
          uint32_t bf[4];
          ldsm_x4_t(vb + (n2 >> 2) * kChunk + key * 128 + unit16 * 16, bf);
          mma_bf16(o[2 * n2], pa, bf[0], bf[1]);
          mma_bf16(o[2 * n2 + 1], pa, bf[2], bf[3]);
        }
      } else {
        pa[0] = pack2_f16(p0[0], p0[1]);
        pa[1] = pack2_f16(p0[2], p0[3]);
        pa[2] = pack2_f16(p1[0], p1[1]);
        pa[3] = pack2_f16(p1[2], p1[3]);
        // Transposed byte-pair matrices (keys 0-7 | 8-15) x (dims of a 16-dim block): a
        // thread gets dims 2r0, 2r0+1 of keys 2q4, 2q4+1; the even and the odd dim make
        // two n8 blocks of the PV product.  o[2B] holds dims 16B + 4q4 + {0, 2}, o[2B+1]
        // dims 16B + 4q4 + {1, 3}.
        const int key = (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
        for (int h32 = 0; h32 < 4; ++h32) {
          const int unit16 = 2 * (h32 & 1) + (lane >> 4);
          uint32_t bf[4];
          ldsm_x4_t(vb + (h32 >> 1) * kChunk + key * 64 + ((unit16 ^ ((key >> 1) & 3)) << 4), bf);
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            const int blk2 = 2 * h32 + hf;
            const uint32_t m_lo = bf[2 * hf], m_hi = bf[2 * hf + 1];  // keys 0-7, keys 8-15
            mma_f16(o[2 * blk2], pa, f16x2_from_e4m3x2(uint16_t(__byte_perm(m_lo, 0, 0x0020))),
                    f16x2_from_e4m3x2(uint16_t(__byte_perm(m_hi, 0, 0x0020))));
            mma_f16(o[2 * blk2 + 1], pa, f16x2_from_e4m3x2(uint16_t(__byte_perm(m_lo, 0, 0x0031))),
                    f16x2_from_e4m3x2(uint16_t(__byte_perm(m_hi, 0, 0x0031))));
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty(st));
    }
    if (!active) continue;

    // ---- the unit's result: row r of the block is draft (16 blk + r) / G, head g G + (16 blk + r) % G
    l_r[0] += __shfl_xor_sync(0xffffffffu, l_r[0], 1);
    l_r[0] += __shfl_xor_sync(0xffffffffu, l_r[0], 2);
    l_r[1] += __shfl_xor_sync(0xffffffffu, l_r[1], 1);
    l_r[1] += __shfl_xor_sync(0xffffffffu, l_r[1], 2);
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      if (draft[half] >= p.q_len) continue;  // padding row
      const int rr = blk * 16 + (half ? r1 : r0);
      const int h = g * G + rr % G;
      const long qrow = long(s) * p.q_len + draft[half];  // query row of (sequence, draft)
      const float M = m_r[half], L = l_r[half];
      if (p.max_splits == 1) {
        float M2 = M, L2 = L, f = 1.f;
        if (p.sink) {
          const float sl = p.sink[h] * kLog2e;
          M2 = fmaxf(M, sl);
          f = ex2(M - M2);
          L2 = L * f + ex2(sl - M2);
        }
        const float sc = p.v_scale * f / L2 * v_deq;
        if constexpr (!FP8) {
          uint32_t* dst = reinterpret_cast<uint32_t*>(p.out + (qrow * kHq + h) * kDv + 2 * q4);
#pragma unroll
          for (int i = 0; i < 16; ++i) dst[i * 4] = pack2_bf16(o[i][2 * half] * sc, o[i][2 * half + 1] * sc);
        } else {
          uint2* dst = reinterpret_cast<uint2*>(p.out + (qrow * kHq + h) * kDv + 4 * q4);
#pragma unroll
          for (int b8 = 0; b8 < 8; ++b8)
            dst[4 * b8] = make_uint2(pack2_bf16(o[2 * b8][2 * half] * sc, o[2 * b8 + 1][2 * half] * sc),
                                     pack2_bf16(o[2 * b8][2 * half + 1] * sc, o[2 * b8 + 1][2 * half + 1] * sc));
        }
        if (p.lse && q4 == 0) p.lse[qrow * kHq + h] = (M2 + __log2f(L2)) * kLn2;
      } else {
        float* dst = p.ws_o + ((qrow * kHq + h) * p.max_splits + split) * kDv;
        if constexpr (!FP8) {
#pragma unroll
          for (int i = 0; i < 16; ++i)
            *reinterpret_cast<float2*>(dst + i * 8 + 2 * q4) = make_float2(o[i][2 * half], o[i][2 * half + 1]);
        } else {
#pragma unroll
          for (int b8 = 0; b8 < 8; ++b8)
            *reinterpret_cast<float4*>(dst + 16 * b8 + 4 * q4) =
                make_float4(o[2 * b8][2 * half] * v_deq, o[2 * b8 + 1][2 * half] * v_deq,
                            o[2 * b8][2 * half + 1] * v_deq, o[2 * b8 + 1][2 * half + 1] * v_deq);
        }
        if (q4 == 0) {
          float* ml = p.ws_ml + ((qrow * kHq + h) * p.max_splits + split) * 2;
          ml[0] = M;
          ml[1] = L;
        }
      }
    }
  }
}

// One warp per (query row, head): merges the split partials and the sink.  A split in which
// a draft row saw no key holds (-inf, 0) and weighs nothing.
__global__ void __launch_bounds__(256) decode_combine_kernel(const __grid_constant__ DecodeParams p) {
  const int wid = int((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (wid >= p.batch * p.q_len * kHq) return;
  const int qrow = wid / kHq, h = wid % kHq;
  const int s = qrow / p.q_len;
  const int ctx = p.seq_lens[s];
  if (ctx < p.q_len) {
    if (lane == 0 && h == 0) atomicOr(p.status, MIMO_STATUS_BAD_INDEX);
    return;
  }
  int nsplit = (ctx - unit_lo(p, ctx) + p.split_len - 1) / p.split_len;
  if (nsplit > p.max_splits) {  // a context beyond max_seq_len: its extra keys were not attended
    if (lane == 0 && h == 0) atomicOr(p.status, MIMO_STATUS_BAD_INDEX);
    nsplit = p.max_splits;
  }
  const float* ml = p.ws_ml + (long(qrow) * kHq + h) * p.max_splits * 2;
  float M = -INFINITY;
  for (int i = lane; i < nsplit; i += 32) M = fmaxf(M, ml[2 * i]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  float sl = -INFINITY;
  if (p.sink) {
    sl = p.sink[h] * kLog2e;
    M = fmaxf(M, sl);
  }
  float L = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  const float* ob = p.ws_o + (long(qrow) * kHq + h) * p.max_splits * kDv;
  for (int i = 0; i < nsplit; ++i) {
    const float w = ex2(ml[2 * i] - M);
    L += w * ml[2 * i + 1];
    const float4 v = *reinterpret_cast<const float4*>(ob + long(i) * kDv + lane * 4);
    acc.x += w * v.x;
    acc.y += w * v.y;
    acc.z += w * v.z;
    acc.w += w * v.w;
  }
  if (p.sink) L += ex2(sl - M);
  const float sc = p.v_scale / L;
  uint2 pk;
  pk.x = pack2_bf16(acc.x * sc, acc.y * sc);
  pk.y = pack2_bf16(acc.z * sc, acc.w * sc);
  *reinterpret_cast<uint2*>(p.out + (long(qrow) * kHq + h) * kDv + lane * 4) = pk;
  if (p.lse && lane == 0) p.lse[long(qrow) * kHq + h] = (M + __log2f(L)) * kLn2;
}

template <bool FP8, int NC>
cudaError_t launch_decode_kernel(const DecodeParams& p, int sms, cudaStream_t s) {
  using Ly = DecodeLayout<FP8, NC>;
  const long units = long(p.batch) * p.hkv * p.n_rp * p.max_splits;
  const long ctas = (units + Ly::kGroups - 1) / Ly::kGroups;
  const int grid = int(ctas < sms ? ctas : sms);
  cudaError_t e = cudaFuncSetAttribute(decode_kernel<FP8, NC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       Ly::kSmemBytes);
  if (e != cudaSuccess) return e;
  decode_kernel<FP8, NC><<<grid, Ly::kThreads, Ly::kSmemBytes, s>>>(p);
  return cudaGetLastError();
}

void decode_rows(int q_len, int group, int* n_blocks, int* nc, int* n_rp) {
  *n_blocks = (q_len * group + 15) / 16;
  *nc = q_len == 1 ? 1 : (*n_blocks <= 2 ? 2 : 4);
  *n_rp = (*n_blocks + *nc - 1) / *nc;
}

cudaError_t launch_decode(const DecodeParams& p, int sms, cudaStream_t s, void* ev_begin, void* ev_end) {
  int nb, nc, n_rp;
  decode_rows(p.q_len, p.group, &nb, &nc, &n_rp);
  if (nb != p.n_blocks || n_rp != p.n_rp || nb * (16 / p.group) > kMaxDrafts) return cudaErrorInvalidValue;
  cudaError_t e;
  if (ev_begin && (e = cudaEventRecord(static_cast<cudaEvent_t>(ev_begin), s)) != cudaSuccess) return e;
  if (p.fp8) {
    e = nc == 1 ? launch_decode_kernel<true, 1>(p, sms, s)
                : (nc == 2 ? launch_decode_kernel<true, 2>(p, sms, s) : launch_decode_kernel<true, 4>(p, sms, s));
  } else {
    e = nc == 1 ? launch_decode_kernel<false, 1>(p, sms, s)
                : (nc == 2 ? launch_decode_kernel<false, 2>(p, sms, s) : launch_decode_kernel<false, 4>(p, sms, s));
  }
  if (e != cudaSuccess) return e;
  if (ev_end && (e = cudaEventRecord(static_cast<cudaEvent_t>(ev_end), s)) != cudaSuccess) return e;
  if (p.max_splits <= 1) return e;
  return launch_decode_combine(p, s);
}

cudaError_t launch_decode_combine(const DecodeParams& p, cudaStream_t s) {
  const long warps = long(p.batch) * p.q_len * kHq;
  decode_combine_kernel<<<unsigned((warps * 32 + 255) / 256), 256, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace mimo
