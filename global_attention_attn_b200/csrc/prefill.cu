// Prefill: varlen causal attention with a sliding window or globally, with or
// without the per-head sink, on the 5th-generation tensor cores.
//
// The layer ("MiMo-V2.6-Flash" miles docs, section 1; "Model techniques map",
// GQA / sliding window / sink / partial RoPE sections):
//   S = scale * rope(Q) rope(K)^T over dims 0..191, masked to the causal window,
//   P = softmax over the row with the sink logit in the denominator,
//   O = v_scale * P V  (V dims 0..127), LSE = ln(sum e^S + e^sink).
//
// Tile shape.  One M tile of 128 MMA rows stacks the G query heads that share a
// KV head (GQA) over R = 128 / G consecutive positions: row m = r * G + h.
//   sliding window (G = 8, R = 16): one key tile of 144 keys covers the window
//     of all 16 positions (positions q0-128 .. q0+15), so 128/144 of the S tile
//     is useful work instead of ~1/2 with 128-position tiles;
//   global (G = 16, R = 8): key tiles of 128 keys aligned to page boundaries
//     (paged caches load one page per tile), online softmax across tiles.
//
// Roles (192 threads): warp 0 issues TMA loads (Q once per M tile, K/V per key
// tile, 128-byte swizzled), warp 1 allocates TMEM and issues tcgen05.mma
// (S = Q K^T into TMEM, double-buffered; O += P V with P read from TMEM), warps
// 2..5 rotate Q in shared memory (partial RoPE fused into the load; the 64
// rotated dims are written back as fp16 and contracted by an fp16 MMA, the 128
// other dims by a bf16 MMA into the same accumulator), run the
// softmax (exp2 domain, running max with rescale only when it grows by more
// than 2^8, sink folded into the initial max and sum), write P into TMEM over
// its S columns, and run the epilogue (O * v_scale / l -> bf16, LSE).
// The global kernel also scores the draft rows of a decode on a paged cache (q_len rows
// per sequence, no cu_seqlens): each sequence's keys are cut into page-aligned splits whose
// partials the decode's combine pass merges.
// Every wait is bounded: a wait that runs out sets MIMO_STATUS_TIMEOUT and the
// CTA unwinds instead of hanging.
#include <cuda_bf16.h>

#include "common.cuh"
#include "ptx.cuh"
#include "../../include/mimoattn.h"

namespace mimo {

namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS1 = 192;
constexpr uint32_t kColO = 384;
constexpr int kThreads = 192;

template <int KIND>
struct Cfg;
template <>
struct Cfg<0> {  // sliding window (prefill_swa_kernel)
  static constexpr int G = 8, R = 16, BN = 144;
};
template <>
struct Cfg<1> {  // global (or any window wider than 129)
  static constexpr int G = 16, R = 8, BN = 128, NQ = 1, NK = 2, NV = 2;
};

constexpr int kMaxSeqs = kPrefillMaxSeqsPerLaunch;  // sequences per launch (the host splits larger batches)

template <int KIND>
struct Layout {
  using C = Cfg<KIND>;
  static constexpr int kQChunk = 128 * 128;          // 128 rows x 64 dims, 2-byte elements
  static constexpr int kQStage = 3 * kQChunk;
  static constexpr int kKChunk = C::BN * 128;
  static constexpr int kKStage = 3 * kKChunk;
  static constexpr int kVChunk = C::BN * 128;
  static constexpr int kVStage = 2 * kVChunk;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + C::NQ * kQStage;
  static constexpr int kOffV = kOffK + C::NK * kKStage;
  static constexpr int kOffBar = kOffV + C::NV * kVStage;
  static constexpr int kNumBars = 3 * C::NQ + 2 * C::NK + 2 * C::NV + 2 + 2 + 1 + 1 + 1 + 1;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kOffSeq = kOffMisc + 16;                       // int [6][kMaxSeqs + 1]
  static constexpr int kOffSink = kOffSeq + 6 * (kMaxSeqs + 1) * 4;   // float [64], log2 units
  static constexpr int kOffCS = (kOffSink + 64 * 4 + 15) / 16 * 16;  // float2 [R][32] cos/sin of a tile
  static constexpr int kBytes = kOffCS + C::R * 32 * 8;
  static_assert(kOffBar % 8 == 0 && kOffSeq % 4 == 0 && kOffCS % 16 == 0, "mbarrier / table / vector alignment");
  static constexpr int kAlloc = kBytes + 1024;  // slack for 1024-byte alignment
  static_assert(kAlloc <= 232448, "shared memory budget");
};

struct TileInfo {
  int s, t, ntiles;          // sequence, tile within it, tiles of the sequence
  int g;                     // kv head
  int q_row0, rows_valid;    // first query row of the tile, valid rows (<= R)
  int qpos0;                 // position of tile row 0
  int key_lo;                // first key position that exists
  int krow_base, kpos_base;  // contiguous key sources: row of position kpos_base
  int new_row0, new_pos0;    // ring-cache chunk: row of the first new key in k / v, its position
  int split;                 // split-KV: the tile's split (key tiles from split * split_tiles), else -1
};

// Per-CTA copy of the per-sequence quantities the roles need for every tile.
struct SeqTable {
  int* tile_start;  // [B + 1] exclusive prefix of M tiles per sequence
  int* q0;          // cu_seqlens_q[s]
  int* qlen;
  int* clen;        // cache_lens[s]
  int* k0;          // cu_seqlens_k[s]
  int* klen;
};

__device__ __forceinline__ SeqTable seq_table(uint8_t* base) {
  int* a = reinterpret_cast<int*>(base);
  constexpr int n = kMaxSeqs + 1;
  return SeqTable{a, a + n, a + 2 * n, a + 3 * n, a + 4 * n, a + 5 * n};
}

// One warp fills the table.
template <int KIND>
__device__ __forceinline__ void fill_seq_table(const PrefillParams& p, const SeqTable& S) {
  constexpr int R = Cfg<KIND>::R;
  const int lane = threadIdx.x & 31;
  int base = 0;
  for (int s0 = 0; s0 < p.num_seqs; s0 += 32) {
    const int s = s0 + lane;
    int n = 0;
    if (s < p.num_seqs) {
      if (KIND == 1 && p.uq > 0) {
        // uq rows (uq <= R: one M tile) ending at the context's last position; with split-KV
        // one work item per split of the context's keys
        const int ql = p.uq, ctx = p.seq_lens[s];
        n = 1;
        if (p.split_tiles > 0) {
          const int len = p.split_tiles * 128;
          n = ctx > 0 ? (ctx - 1) / len + 1 : 0;
          if (n > p.max_splits) {  // a context beyond max_seq_len: its extra keys are not attended
            atomicOr(p.status, MIMO_STATUS_BAD_INDEX);
            n = p.max_splits;
          }
        }
        if (ctx < ql) {  // fewer positions than query rows: nothing to attend
          atomicOr(p.status, MIMO_STATUS_BAD_INDEX);
          n = 0;
        }
        S.q0[s] = (p.seq_base + s) * ql;
        S.qlen[s] = ql;
        S.clen[s] = ctx;  // as for a paged prefill: every key, the drafts included, is in the cache
        S.k0[s] = 0;
        S.klen[s] = 0;
      } else {
        const int q0 = p.cu_q[s], ql = p.cu_q[s + 1] - q0;
        n = (ql + R - 1) / R;
        S.q0[s] = q0;
        S.qlen[s] = ql;
        S.clen[s] = p.cache_lens ? p.cache_lens[s] : 0;
        S.k0[s] = p.cu_k ? p.cu_k[s] : 0;
        S.klen[s] = p.cu_k ? p.cu_k[s + 1] - p.cu_k[s] : 0;
      }
    }
    int incl = n;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (s < p.num_seqs) S.tile_start[s] = base + incl - n;
    base += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (lane == 0) S.tile_start[p.num_seqs] = base;
}

// Maps work item w to (sequence, tile, kv head) from the shared table; any
// thread may call it.  Tiles of a sequence are ordered longest-first for
// global attention, in snake order over the rounds of the persistent grid.
template <int KIND>
__device__ __forceinline__ bool locate(const PrefillParams& p, const SeqTable& S, int w, TileInfo& T) {
  constexpr int R = Cfg<KIND>::R;
  const int total = S.tile_start[p.num_seqs] * p.hkv;
  if (w >= total) return false;
  if (KIND != 0) {
    // CTA i takes items i, i + grid, ...: reverse every other round of grid items, so the
    // CTA that gets a round's longest tile gets the next round's shortest
    const int G = int(gridDim.x), round = w / G, base = round * G;
    if (round & 1) w = base + min(G, total - base) - 1 - (w - base);
  }
  const int tt = w / p.hkv;
  int lo = 0, hi = p.num_seqs;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (S.tile_start[mid] <= tt) lo = mid; else hi = mid;
  }
  T.s = lo;
  T.ntiles = S.tile_start[lo + 1] - S.tile_start[lo];
  int t = tt - S.tile_start[lo];
  T.split = -1;
  if (KIND == 1 && p.split_tiles > 0) {  // items of a sequence are the splits of its one M tile
    T.split = t;
    T.ntiles = 1;
    t = 0;
  } else if (KIND != 0) {
    t = T.ntiles - 1 - t;
  }
  T.t = t;
  T.g = w % p.hkv;
  const int qlen = S.qlen[lo], clen = S.clen[lo];
  const int ctx = clen + S.klen[lo];
  T.q_row0 = S.q0[lo] + t * R;
  T.rows_valid = min(R, qlen - t * R);
  T.qpos0 = ctx - qlen + t * R;
  if (p.mode == kModeContig) {
    T.key_lo = clen;
    T.krow_base = S.k0[lo];
    T.kpos_base = clen;
  } else if (p.mode == kModeExt) {
    T.key_lo = max(0, clen - 128);
    T.krow_base = S.k0[lo] + 128 * (p.seq_base + lo);
    T.kpos_base = clen - 128;
    T.new_row0 = S.k0[lo];
    T.new_pos0 = clen;
  } else {
    T.key_lo = 0;
    T.krow_base = 0;
    T.kpos_base = 0;
  }
  return true;
}

// Key tiles of an M tile: [j_lo, j_lo + n) with tile j starting at position key_tile_start(j).
template <int KIND>
__device__ __forceinline__ void key_tiles(const PrefillParams& p, const TileInfo& T, int* j_lo, int* n) {
  if (KIND == 0) {
    *j_lo = 0;
    *n = 1;
  } else {
    const int qlast = T.qpos0 + max(T.rows_valid, 1) - 1;
    const int lo = p.window > 0 ? max(0, T.qpos0 - p.window + 1) : 0;
    *j_lo = max(lo, 0) / 128;
    *n = max(qlast, 0) / 128 - *j_lo + 1;
    if (T.split >= 0) {  // this split's share; at least one tile (its keys are masked if none is visible)
      const int a = T.split * p.split_tiles;
      const int e = min(*j_lo + *n, a + p.split_tiles);
      *j_lo = max(*j_lo, a);
      *n = max(e - *j_lo, 1);
    }
  }
}
template <int KIND>
__device__ __forceinline__ int key_tile_start(const TileInfo& T, int j) {
  return KIND == 0 ? T.qpos0 - 128 : j * 128;
}

}  // namespace

// SPLIT: the draft-row mode's split-KV partials (p.split_tiles > 0); a separate instance, so
// the prefill's own code carries none of it
template <int KIND, bool SPLIT>
__global__ void __launch_bounds__(kThreads, 1) prefill_kernel(const __grid_constant__ PrefillParams p) {
  using C = Cfg<KIND>;
  using Ly = Layout<KIND>;
  constexpr int G = C::G, R = C::R, BN = C::BN, NQ = C::NQ, NK = C::NK, NV = C::NV;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // barrier addresses
  const uint32_t bar0 = sbase + Ly::kOffBar;
  auto q_full = [&](int i) { return bar0 + 8 * i; };
  auto q_rot = [&](int i) { return bar0 + 8 * (NQ + i); };
  auto q_empty = [&](int i) { return bar0 + 8 * (2 * NQ + i); };
  auto k_full = [&](int i) { return bar0 + 8 * (3 * NQ + i); };
  auto k_empty = [&](int i) { return bar0 + 8 * (3 * NQ + NK + i); };
  auto v_full = [&](int i) { return bar0 + 8 * (3 * NQ + 2 * NK + i); };
  auto v_empty = [&](int i) { return bar0 + 8 * (3 * NQ + 2 * NK + NV + i); };
  auto s_full = [&](int i) { return bar0 + 8 * (3 * NQ + 2 * NK + 2 * NV + i); };
  auto p_full = [&](int i) { return bar0 + 8 * (3 * NQ + 2 * NK + 2 * NV + 2 + i); };
  const uint32_t pv_done = bar0 + 8 * (3 * NQ + 2 * NK + 2 * NV + 4);
  const uint32_t o_empty = pv_done + 8;
  const uint32_t drain = pv_done + 16;
  const uint32_t cs_ready = pv_done + 24;  // the softmax warps' cos/sin table is written
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Ly::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Ly::kOffMisc + 4);
  const SeqTable S = seq_table(smem + Ly::kOffSeq);
  float* sink_l2 = reinterpret_cast<float*>(smem + Ly::kOffSink);
  float2* cs = reinterpret_cast<float2*>(smem + Ly::kOffCS);

  if (threadIdx.x == 0) {
    for (int i = 0; i < NQ; ++i) {
      mbar_init(q_full(i), 1);
      mbar_init(q_rot(i), 128);
      mbar_init(q_empty(i), 1);
    }
    for (int i = 0; i < NK; ++i) {
      mbar_init(k_full(i), 1);
      mbar_init(k_empty(i), 1);
    }
    for (int i = 0; i < NV; ++i) {
      mbar_init(v_full(i), 1);
      mbar_init(v_empty(i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(s_full(i), 1);
      mbar_init(p_full(i), 128);
    }
    mbar_init(pv_done, 1);
    mbar_init(o_empty, 128);
    mbar_init(drain, 1);
    mbar_init(cs_ready, 128);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) fill_seq_table<KIND>(p, S);
  if (warp == 1) {
    tmem_alloc(smem_addr(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  if (threadIdx.x >= 64 && threadIdx.x < 128)
    sink_l2[threadIdx.x - 64] = p.sink ? p.sink[threadIdx.x - 64] * kLog2e : -INFINITY;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  unsigned* status = p.status;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producers
    // lane 0 streams Q tiles, lane 1 K tiles, lane 2 V tiles, each at its own pace.
    if (lane < 3) {
      if (lane == 0) {
        tma_prefetch(&p.tm_q);
        tma_prefetch(&p.tm_k0);
        tma_prefetch(&p.tm_k12);
        tma_prefetch(&p.tm_v);
      }
      // the rotated key copies come from the key pre-pass, which may still be running
      pdl_wait_prerequisites();
      int mt = 0, jj = 0;
      bool ok = true;
      for (int w = blockIdx.x; ok; w += gridDim.x) {
        TileInfo T;
        if (!locate<KIND>(p, S, w, T)) break;
        if (lane == 0) {
          if (p.withhold_q) break;  // failure-detection test: no query tile ever arrives
          const int qs = mt % NQ;
          if (mt >= NQ) ok = mbar_wait(q_empty(qs), ((mt / NQ) - 1) & 1, abort_flag, status, MIMO_STATUS_TIMEOUT, p.wait_ns);
          if (!ok) break;
          const uint32_t qdst = sbase + Ly::kOffQ + qs * Ly::kQStage;
          mbar_expect_tx(q_full(qs), Ly::kQStage);
          for (int c = 0; c < 3; ++c)
            tma_load_3d(qdst + c * Ly::kQChunk, &p.tm_q, q_full(qs), 64 * c, T.g * G, T.q_row0);
        } else {
          int j_lo, nkv;
          key_tiles<KIND>(p, T, &j_lo, &nkv);
          for (int j = 0; j < nkv && ok; ++j, ++jj) {
            const int kt0 = key_tile_start<KIND>(T, j_lo + j);
            int row;
            if (p.mode == kModePaged) {
              const int pi = j_lo + j;
              int page = pi < p.max_pages ? p.block_table[long(T.s) * p.max_pages + pi] : -1;
              if (page < 0 || page >= p.num_pages) {
                if (lane == 1) atomicOr(status, MIMO_STATUS_BAD_INDEX);
                page = 0;
              }
              row = page * 128;
            } else {
              row = T.krow_base + (kt0 - T.kpos_base);
            }
            if (lane == 1) {
              const int ks = jj % NK;
              if (jj >= NK) ok = mbar_wait(k_empty(ks), ((jj / NK) - 1) & 1, abort_flag, status, MIMO_STATUS_TIMEOUT, p.wait_ns);
              if (!ok) break;
              const uint32_t kdst = sbase + Ly::kOffK + ks * Ly::kKStage;
              mbar_expect_tx(k_full(ks), Ly::kKStage);
              tma_load_3d(kdst, &p.tm_k0, k_full(ks), 0, T.g, row);
              tma_load_3d(kdst + Ly::kKChunk, &p.tm_k12, k_full(ks), 64, T.g, row);
              tma_load_3d(kdst + 2 * Ly::kKChunk, &p.tm_k12, k_full(ks), 128, T.g, row);
            } else {
              const int vs = jj % NV;
              if (jj >= NV) ok = mbar_wait(v_empty(vs), ((jj / NV) - 1) & 1, abort_flag, status, MIMO_STATUS_TIMEOUT, p.wait_ns);
              if (!ok) break;
              const uint32_t vdst = sbase + Ly::kOffV + vs * Ly::kVStage;
              mbar_expect_tx(v_full(vs), Ly::kVStage);
              tma_load_3d(vdst, &p.tm_v, v_full(vs), 0, T.g, row);
              tma_load_3d(vdst + Ly::kVChunk, &p.tm_v, v_full(vs), 64, T.g, row);
            }
          }
        }
        ++mt;
      }
      if (!ok) {
        // let copies already in flight land before the CTA leaves
        int dummy = 0;
        for (int i = 0; i < NQ; ++i) mbar_wait(q_full(i), 0, &dummy, nullptr, 0, 50000000ull);
        for (int i = 0; i < NK; ++i) mbar_wait(k_full(i), 0, &dummy, nullptr, 0, 50000000ull);
        for (int i = 0; i < NV; ++i) mbar_wait(v_full(i), 0, &dummy, nullptr, 0, 50000000ull);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (lane 0)
    // Issue order over the continuous stream of key tiles: QK(jj), then PV(jj-1),
    // so the next M tile's QK^T runs while the current tile's softmax finishes.
    if (lane == 0) {
      constexpr uint32_t idesc_qk_rot = idesc_f32acc(128, BN, 0, 0, 0);  // dims 0..63: fp16 x fp16
      constexpr uint32_t idesc_qk = idesc_f32acc(128, BN, 0, 0, 1);      // dims 64..191: bf16 x bf16
      constexpr uint32_t idesc_pv = idesc_f32acc(128, 128, 0, 1, 1);
      int mt = 0, jj = 0;
      bool ok = true;
      int pend_jj = -1, pend_mt = 0;
      bool pend_first = false;
      auto issue_pv = [&](int jp, bool first, int mtp) -> bool {
        const int b = jp & 1;
        if (!mbar_wait(p_full(b), (jp >> 1) & 1, abort_flag, status, MIMO_STATUS_TIMEOUT, p.wait_ns)) return false;
        const int vs = jp % NV;
        if (!mbar_wait(v_full(vs), (jp / NV) & 1, abort_flag, status, MIMO_STATUS_TIMEOUT, p.wait_ns)) return false;
        if (first && mtp > 0 && !mbar_wait(o_empty, (mtp - 1) & 1, abort_flag, status, MIMO_STATUS_TIMEOUT, p.wait_ns))
          return false;
        tc_fence_after();
        const uint32_t vbase = sbase + Ly::kOffV + vs * Ly::kVStage;
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          const uint64_t bd = sdesc_sw128(vbase + kk * 2048, Ly::kVChunk, 1024);
          tc_mma_ts(tmem + kColO, tmem + b * kColS1 + kk * 8, bd, idesc_pv, (first && kk == 0) ? 0u : 1u);
        }
        tc_commit(v_empty(vs));
        tc_commit(pv_done);
        return true;
      };
      for (int w = blockIdx.x; ok; w += gridDim.x) {
        TileInfo T;
        if (!locate<KIND>(p, S, w, T)) break;
        const int qs = mt % NQ;
        if (!(ok = mbar_wait(q_rot(qs), (mt / NQ) & 1, abort_flag, status, MIMO_STATUS_TIMEOUT, p.wait_ns))) break;
        tc_fence_after();
        int j_lo, nkv;
        key_tiles<KIND>(p, T, &j_lo, &nkv);
        const uint32_t qbase = sbase + Ly::kOffQ + qs * Ly::kQStage;
        for (int j = 0; j < nkv; ++j) {
          const int ks = jj % NK;
          if (!(ok = mbar_wait(k_full(ks), (jj / NK) & 1, abort_flag, status, MIMO_STATUS_TIMEOUT, p.wait_ns))) break;
          tc_fence_after();
          const int b = jj & 1;
          const uint32_t kbase = sbase + Ly::kOffK + ks * Ly::kKStage;
#pragma unroll
          for (int c = 0; c < 3; ++c)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t ad = sdesc_sw128(qbase + c * Ly::kQChunk + kk * 32, 16, 1024);
              const uint64_t bd = sdesc_sw128(kbase + c * Ly::kKChunk + kk * 32, 16, 1024);
              tc_mma_ss(tmem + b * kColS1, ad, bd, c == 0 ? idesc_qk_rot : idesc_qk, (c | kk) ? 1u : 0u);
            }
          tc_commit(s_full(b));
          tc_commit(k_empty(ks));
          if (j == nkv - 1) tc_commit(q_empty(qs));
          if (pend_jj >= 0 && !(ok = issue_pv(pend_jj, pend_first, pend_mt))) break;
          pend_jj = jj;
          pend_first = (j == 0);
          pend_mt = mt;
          ++jj;
        }
        if (!ok) break;
        ++mt;
      }
      if (ok && pend_jj >= 0) ok = issue_pv(pend_jj, pend_first, pend_mt);
      if (!ok) {
        int dummy = 0;
        tc_commit(drain);
        mbar_wait(drain, 0, &dummy, nullptr, 0, 50000000ull);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ RoPE + softmax + epilogue
    const int tid = threadIdx.x - 64;  // 0..127
    const int quad = warp & 3;
    const int m = quad * 32 + lane;  // TMEM lane = M row
    const int r = m / G, hq = m % G;
    const uint32_t t_lane = tmem + (uint32_t(quad * 32) << 16);
    const float c_log2 = p.scale_log2;

    // The four softmax warps take every decision together: a wait that fails in one
    // lane fails for the whole warp, so warp-collective tcgen05 ops never diverge.
    auto wait_w = [&](uint32_t bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, status, MIMO_STATUS_TIMEOUT, p.wait_ns));
    };
    int n_rot = 0;
    // Partial RoPE of M tile T in Q stage qs: the R x 32 cos/sin pairs are computed
    // once per tile (the G heads of a position share them), then each thread
    // rotates dims 0..63 of its row in place (128-byte swizzled rows) to fp16.
    // The table is free to overwrite here: every thread read the previous one
    // before arriving on q_rot, and this thread passed an s_full since.
    auto rotate_q = [&](const TileInfo& T, int qs) -> bool {
#pragma unroll
      for (int e = tid; e < R * 32; e += 128) {
        const int rr = e >> 5, j = e & 31;
        const int pos = rr < T.rows_valid ? T.qpos0 + rr : 0;
        float c, s;
        rope_cos_sin(pos, p.rope.inv_freq[j], &c, &s);
        cs[e] = make_float2(c, s);
      }
      mbar_arrive(cs_ready);
      if (!wait_w(cs_ready, n_rot & 1)) return false;
      ++n_rot;
      uint8_t* row = smem + Ly::kOffQ + qs * Ly::kQStage + m * 128;
      const int sw = m & 7;
      const float2* csr = cs + r * 32;
      float amax = 0.f;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        uint4* plo = reinterpret_cast<uint4*>(row + ((u ^ sw) << 4));
        uint4* phi = reinterpret_cast<uint4*>(row + (((u + 4) ^ sw) << 4));
        uint4 lo = *plo, hi = *phi;
        rope_chunk_pair_cs(lo, hi, csr + 8 * u, amax);
        *plo = lo;
        *phi = hi;
      }
      if (amax > kF16Max && r < T.rows_valid) atomicOr(status, MIMO_STATUS_RANGE);
      fence_proxy_async_smem();
      mbar_arrive(q_rot(qs));
      return true;
    };

    int mt = 0, jj = 0;
    bool ok = true;
    int w = blockIdx.x;
    TileInfo T;
    bool have = locate<KIND>(p, S, w, T);
    if (have) ok = wait_w(q_full(0), 0) && rotate_q(T, 0);
    while (have && ok) {
      const bool row_valid = r < T.rows_valid;
      const int qp = T.qpos0 + r;
      const int head = T.g * G + hq;
      // a split's partial leaves the sink to the combine pass
      float m_run = SPLIT ? -INFINITY : sink_l2[head];
      float l_run = (p.sink && !SPLIT) ? 1.f : 0.f;
      // visible key positions of this row: [vis_lo, vis_hi]
      const int vis_hi = row_valid ? qp : -0x40000000;
      const int vis_lo = max(T.key_lo, p.window > 0 ? qp - p.window + 1 : -0x40000000);
      int j_lo, nkv;
      key_tiles<KIND>(p, T, &j_lo, &nkv);
      const int qlast = T.qpos0 + T.rows_valid - 1;
      for (int j = 0; j < nkv; ++j) {
        const int b = jj & 1;
        if (!(ok = wait_w(s_full(b), (jj >> 1) & 1))) break;
        tc_fence_after();
        uint32_t sr[BN];
#pragma unroll
        for (int c = 0; c + 32 <= BN; c += 32) tmem_ld32(t_lane + b * kColS1 + c, sr + c);
        if (BN % 32) tmem_ld16(t_lane + b * kColS1 + (BN / 32) * 32, sr + (BN / 32) * 32);
        static_assert(BN == 128, "the wait below binds 128 registers");
        tmem_wait_ld_r64(sr);
        tmem_wait_ld_r64(sr + 64);
        float* sv = reinterpret_cast<float*>(sr);
        const int kt0 = key_tile_start<KIND>(T, j_lo + j);
        const bool interior = kt0 >= T.key_lo && kt0 + BN - 1 <= T.qpos0 &&
                              (p.window <= 0 || qlast - kt0 < p.window) && T.rows_valid == R;
        float mx = -INFINITY;
        if (interior) {
#pragma unroll
          for (int c = 0; c < BN; ++c) mx = fmaxf(mx, sv[c]);
        } else {
          const int a = vis_lo - kt0, e = vis_hi - kt0;
#pragma unroll
          for (int c = 0; c < BN; ++c) {
            if (c < a || c > e) sv[c] = -INFINITY;
            mx = fmaxf(mx, sv[c]);
          }
        }
        const float mt_l2 = mx * c_log2;
        const float m_new = fmaxf(m_run, mt_l2);
        float alpha = 1.f;
        const bool resc = m_new > m_run + 8.f;
        if (resc) {
          alpha = ex2(m_run - m_new);
          m_run = m_new;
        }
        // Only a rescale of O needs PV(j-1) to have landed: P(j) goes to the other S buffer,
        // whose previous P was read by PV(j-2), which completed before QK(j) (in-order MMAs).
        if (__any_sync(0xffffffffu, resc && j > 0)) {
          if (!(ok = wait_w(pv_done, (jj - 1) & 1))) break;
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < 128; c += 32) {
            uint32_t o[32];
            tmem_ld32(t_lane + kColO + c, o);
            tmem_wait_ld_r32(o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st16(t_lane + kColO + c, o);
            tmem_st16(t_lane + kColO + c + 16, o + 16);
          }
        }
        l_run *= alpha;
        const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
        float lsum = 0.f;
#pragma unroll
        for (int c = 0; c < BN; c += 2) {
          const float p0 = ex2(fmaf(sv[c], c_log2, -m_use));
          const float p1 = ex2(fmaf(sv[c + 1], c_log2, -m_use));
          lsum += p0 + p1;
          sr[c / 2] = pack_bf16x2(p0, p1);
        }
        l_run += lsum;
#pragma unroll
        for (int c = 0; c + 16 <= BN / 2; c += 16) tmem_st16(t_lane + b * kColS1 + c, sr + c);
        if ((BN / 2) % 16) tmem_st8(t_lane + b * kColS1 + (BN / 2 / 16) * 16, sr + (BN / 2 / 16) * 16);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(p_full(b));
        ++jj;
      }
      if (!ok) break;
      // ---- rotate the next tile's Q before this tile's epilogue, so its QK^T overlaps
      w += gridDim.x;
      TileInfo Tn;
      const bool have_next = locate<KIND>(p, S, w, Tn);
      if (have_next) {
        const int qs = (mt + 1) % NQ;
        if (!(ok = wait_w(q_full(qs), ((mt + 1) / NQ) & 1) && rotate_q(Tn, qs))) break;
      }
      // ---- epilogue: O is final once the PVs of this tile's last two key tiles landed.
      // The softmax waits for a PV only when it rescales O, so both may still be pending
      // here, and a single parity wait could be met by the phase before them: wait in order.
      if (nkv >= 2 && !(ok = wait_w(pv_done, (jj - 2) & 1))) break;
      if (!(ok = wait_w(pv_done, (jj - 1) & 1))) break;
      tc_fence_after();
      if constexpr (SPLIT) {
        // split-KV partial: O as accumulated (relative to m_run), with (m_run, l_run)
        const long pr = (long(T.q_row0 + r) * kHq + head) * p.max_splits + T.split;
        float* dst = p.ws_o + pr * kDv;
        // the whole row of O in one load round trip
        uint32_t o[128];
#pragma unroll
        for (int c = 0; c < 128; c += 32) tmem_ld32(t_lane + kColO + c, o + c);
        tmem_wait_ld_r64(o);
        tmem_wait_ld_r64(o + 64);
        if (row_valid) {
          uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
          for (int i = 0; i < 32; ++i) d4[i] = make_uint4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
        }
        if (row_valid) *reinterpret_cast<float2*>(p.ws_ml + 2 * pr) = make_float2(m_run, l_run);
        tc_fence_before();
        mbar_arrive(o_empty);
        ++mt;
        T = Tn;
        have = have_next;
        continue;
      }
      const float sc = p.v_scale / l_run;
      uint16_t* orow = p.out + (long(T.q_row0 + r) * kHq + head) * kDv;
      // the whole row of O in one load round trip
      uint32_t oall[128];
#pragma unroll
      for (int c = 0; c < 128; c += 32) tmem_ld32(t_lane + kColO + c, oall + c);
      tmem_wait_ld_r64(oall);
      tmem_wait_ld_r64(oall + 64);
#pragma unroll
      for (int c = 0; c < 128; c += 32) {
        const uint32_t* o = oall + c;
        uint4 pk[4];
        uint32_t* w32 = reinterpret_cast<uint32_t*>(pk);
#pragma unroll
        for (int i = 0; i < 16; ++i)
          w32[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * sc, __uint_as_float(o[2 * i + 1]) * sc);
        if (row_valid) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c);
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i] = pk[i];
        }
      }
      if (row_valid && p.lse) p.lse[long(T.q_row0 + r) * kHq + head] = (m_run + __log2f(l_run)) * kLn2;
      tc_fence_before();
      mbar_arrive(o_empty);
      ++mt;
      T = Tn;
      have = have_next;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------- sliding window
// The sliding-window layer (window <= 129) has exactly one 144-key tile per M
// tile, so there is no loop over key tiles to pipeline.  Instead two softmax
// warpgroups take alternate M tiles (WG0 the even ones, WG1 the odd ones) and
// work on them at the same time.  Each tile owns a 256-column TMEM region:
// S in columns 0..143, then P (bf16 pairs) over columns 0..71 and O in columns
// 72..199, which only holds S values the softmax has already read.  Warps 10
// and 11 apply the partial RoPE to each Q tile in shared memory, with a
// per-row (cos, sin) table that the key pre-pass computes once per query row.  With 12
// warps, each SM sub-partition holds 3, which caps registers at 168 per
// thread.  The code each softmax warp runs once per tile is kept short: the kernel's
// roles run different code at the same time, and instruction fetch, not the exponential
// unit, set the softmax's pace (the same S columns 32..127 go through one copy of a
// 32-column loop body, and the epilogue's four O chunks through one).  The MMA
// lane issues QK^T of tile t before PV of tile t-1; QK^T of tile t waits until
// the epilogue of tile t-2 (same region) has read O.
namespace {
struct SwaLayout {
  using C = Cfg<0>;
  static constexpr int kQChunk = 128 * 128;
  static constexpr int kQStage = 3 * kQChunk;
  static constexpr int kKChunk = C::BN * 128;
  static constexpr int kVChunk = C::BN * 128;
  static constexpr int kOffQ = 0;                          // 2 stages
  static constexpr int kOffK = kOffQ + 2 * kQStage;         // 1 stage, 3 chunks
  static constexpr int kOffV = kOffK + 3 * kKChunk;         // 1 stage, 2 chunks
  static constexpr int kOffBar = kOffV + 2 * kVChunk;
  static constexpr int kNumBars = 24;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kOffSeq = kOffMisc + 16;
  static constexpr int kOffSink = kOffSeq + 6 * (kMaxSeqs + 1) * 4;
  static constexpr int kOffCS = (kOffSink + 64 * 4 + 1023) / 1024 * 1024;  // float2 [2][R][32] per Q stage (TMA)
  static constexpr int kCSStage = C::R * 32 * 8;
  static constexpr int kOffStage = kOffCS + 2 * kCSStage;  // O staging: 8 softmax warps x 32 rows x 64 bytes
  static constexpr int kStageBytes = 32 * 64;
  static constexpr int kBytes = kOffStage + 8 * kStageBytes;
  static constexpr int kAlloc = kBytes + 1024;
  static_assert(kAlloc <= 232448, "shared memory budget");
  static_assert(kOffBar % 8 == 0 && kOffSeq % 4 == 0 && kOffStage % 16 == 0, "mbarrier / table / vector alignment");
  static_assert(kOffCS % 128 == 0 && kOffQ % 1024 == 0 && kOffK % 1024 == 0 && kOffV % 1024 == 0,
                "TMA destinations: 1024-byte aligned for 128-byte swizzle, 128-byte otherwise");
};
constexpr int kSwaThreads = 384;
constexpr uint32_t kSwaRegion = 256;  // TMEM columns per tile region
constexpr uint32_t kSwaColO = 72;     // O inside a region
}  // namespace

__global__ void __launch_bounds__(kSwaThreads, 1) prefill_swa_kernel(const __grid_constant__ PrefillParams p) {
  using C = Cfg<0>;
  using Ly = SwaLayout;
  constexpr int G = C::G, BN = C::BN;
  constexpr int CH = BN / 3;  // 48 columns per softmax chunk
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const uint32_t bar0 = sbase + Ly::kOffBar;
  auto q_full = [&](int b) { return bar0 + 8 * (0 + b); };
  auto q_rot = [&](int b) { return bar0 + 8 * (2 + b); };
  auto q_empty = [&](int b) { return bar0 + 8 * (4 + b); };
  const uint32_t k_full = bar0 + 8 * 6, k_empty = bar0 + 8 * 7, v_full = bar0 + 8 * 8, v_empty = bar0 + 8 * 9;
  auto s_full = [&](int b) { return bar0 + 8 * (10 + b); };
  auto p_full = [&](int b) { return bar0 + 8 * (12 + b); };
  auto pv_done = [&](int b) { return bar0 + 8 * (14 + b); };
  auto o_empty = [&](int b) { return bar0 + 8 * (16 + b); };
  const uint32_t drain = bar0 + 8 * 20;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Ly::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Ly::kOffMisc + 4);
  const SeqTable S = seq_table(smem + Ly::kOffSeq);
  float* sink_l2 = reinterpret_cast<float*>(smem + Ly::kOffSink);

  if (threadIdx.x == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(q_full(b), 1);
      mbar_init(q_rot(b), 64);
      mbar_init(q_empty(b), 1);
      mbar_init(s_full(b), 1);
      mbar_init(p_full(b), 128);
      mbar_init(pv_done(b), 1);
      mbar_init(o_empty(b), 128);
    }

    mbar_init(k_full, 1);
    mbar_init(k_empty, 1);
    mbar_init(v_full, 1);
    mbar_init(v_empty, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) fill_seq_table<0>(p, S);
  if (warp == 1) {
    tmem_alloc(smem_addr(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  if (threadIdx.x >= 64 && threadIdx.x < 128)
    sink_l2[threadIdx.x - 64] = p.sink ? p.sink[threadIdx.x - 64] * kLog2e : -INFINITY;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  unsigned* status = p.status;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producers (Q, K, V lanes)
    if (lane < 3) {
      if (lane == 0) {
        tma_prefetch(&p.tm_q);
        tma_prefetch(&p.tm_k0);
        tma_prefetch(&p.tm_k12);
        tma_prefetch(&p.tm_v);
        tma_prefetch(&p.tm_cs);
        if (p.mode == kModeExt) {
          tma_prefetch(&p.tm_k0n);
          tma_prefetch(&p.tm_k12n);
          tma_prefetch(&p.tm_vn);
        }
      }
      // the rotated key copies and the cos/sin rows come from the key pre-pass, which may
      // still be running: everything before this point (barriers, tensor memory, the
      // sequence table) overlapped it
      pdl_wait_prerequisites();
      bool ok = true;
      int mt = 0;
      for (int w = blockIdx.x; ok; w += gridDim.x, ++mt) {
        TileInfo T;
        if (!locate<0>(p, S, w, T)) break;
        // a ring-cache chunk's tile whose window starts inside the chunk reads the new keys
        // directly; the others (and every other mode) read the rows T.krow_base refers to
        const int kt0 = T.qpos0 - 128;
        const bool direct = p.mode == kModeExt && kt0 >= T.new_pos0;
        const int row = direct ? T.new_row0 + (kt0 - T.new_pos0) : T.krow_base + (kt0 - T.kpos_base);
        const CUtensorMap* mk0 = direct ? &p.tm_k0n : &p.tm_k0;
        const CUtensorMap* mk12 = direct ? &p.tm_k12n : &p.tm_k12;
        const CUtensorMap* mv = direct ? &p.tm_vn : &p.tm_v;
        if (lane == 0) {
          if (p.withhold_q) break;  // failure-detection test: no query tile ever arrives
          const int b = mt & 1;
          if (mt >= 2 && !(ok = mbar_wait(q_empty(b), ((mt >> 1) - 1) & 1, abort_flag, status, MIMO_STATUS_TIMEOUT, p.wait_ns)))
            break;
          const uint32_t qdst = sbase + Ly::kOffQ + b * Ly::kQStage;
          mbar_expect_tx(q_full(b), Ly::kQStage + Ly::kCSStage);
          for (int c = 0; c < 3; ++c)
            tma_load_3d(qdst + c * Ly::kQChunk, &p.tm_q, q_full(b), 64 * c, T.g * G, T.q_row0);
          tma_load_2d(sbase + Ly::kOffCS + b * Ly::kCSStage, &p.tm_cs, q_full(b), 0, T.q_row0);
        } else if (lane == 1) {
          if (mt >= 1 && !(ok = mbar_wait(k_empty, (mt - 1) & 1, abort_flag, status, MIMO_STATUS_TIMEOUT, p.wait_ns))) break;
          const uint32_t kdst = sbase + Ly::kOffK;
          mbar_expect_tx(k_full, 3 * Ly::kKChunk);
          tma_load_3d(kdst, mk0, k_full, 0, T.g, row);
          tma_load_3d(kdst + Ly::kKChunk, mk12, k_full, 64, T.g, row);
          tma_load_3d(kdst + 2 * Ly::kKChunk, mk12, k_full, 128, T.g, row);
        } else {
          if (mt >= 1 && !(ok = mbar_wait(v_empty, (mt - 1) & 1, abort_flag, status, MIMO_STATUS_TIMEOUT, p.wait_ns))) break;
          const uint32_t vdst = sbase + Ly::kOffV;
          mbar_expect_tx(v_full, 2 * Ly::kVChunk);
          tma_load_3d(vdst, mv, v_full, 0, T.g, row);
          tma_load_3d(vdst + Ly::kVChunk, mv, v_full, 64, T.g, row);
        }
      }
      if (!ok) {
        int dummy = 0;
        for (int b = 0; b < 2; ++b) mbar_wait(q_full(b), 0, &dummy, nullptr, 0, 50000000ull);
        mbar_wait(k_full, 0, &dummy, nullptr, 0, 50000000ull);
        mbar_wait(v_full, 0, &dummy, nullptr, 0, 50000000ull);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (lane 0)
    if (lane == 0) {
      constexpr uint32_t idesc_qk_rot = idesc_f32acc(128, BN, 0, 0, 0);  // dims 0..63: fp16 x fp16
      constexpr uint32_t idesc_qk = idesc_f32acc(128, BN, 0, 0, 1);      // dims 64..191: bf16 x bf16
      constexpr uint32_t idesc_pv = idesc_f32acc(128, 128, 0, 1, 1);
      bool ok = true;
      auto issue_pv = [&](int t) -> bool {
        const int b = t & 1;
        if (!mbar_wait(p_full(b), (t >> 1) & 1, abort_flag, status, MIMO_STATUS_TIMEOUT, p.wait_ns)) return false;
        if (!mbar_wait(v_full, t & 1, abort_flag, status, MIMO_STATUS_TIMEOUT, p.wait_ns)) return false;
        tc_fence_after();
        const uint32_t reg = tmem + b * kSwaRegion;
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          const uint64_t bd = sdesc_sw128(sbase + Ly::kOffV + kk * 2048, Ly::kVChunk, 1024);
          tc_mma_ts(reg + kSwaColO, reg + kk * 8, bd, idesc_pv, kk == 0 ? 0u : 1u);
        }
        tc_commit(v_empty);
        tc_commit(pv_done(b));
        return true;
      };
      // Two cursors: tq = next tile to multiply QK^T for, tp = next tile to multiply PV
      // for (tp <= tq <= tp + 1: two TMEM regions).  Whichever is ready goes first, so
      // one warpgroup's PV never waits on the other warpgroup's next Q.
      auto issue_qk = [&](int t) {
        const int b = t & 1;
        tc_fence_after();
        const uint32_t qbase = sbase + Ly::kOffQ + b * Ly::kQStage;
        const uint32_t kbase = sbase + Ly::kOffK;
#pragma unroll
        for (int c = 0; c < 3; ++c)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = sdesc_sw128(qbase + c * Ly::kQChunk + kk * 32, 16, 1024);
            const uint64_t bd = sdesc_sw128(kbase + c * Ly::kKChunk + kk * 32, 16, 1024);
            tc_mma_ss(tmem + b * kSwaRegion, ad, bd, c == 0 ? idesc_qk_rot : idesc_qk, (c | kk) ? 1u : 0u);
          }
        tc_commit(s_full(b));
        tc_commit(k_empty);
        tc_commit(q_empty(b));
      };
      int tq = 0, tp = 0;
      bool have_q;
      {
        TileInfo T;
        have_q = locate<0>(p, S, blockIdx.x, T);
      }
      uint64_t t_last = global_timer_ns();
      while (have_q || tp < tq) {
        bool progress = false;
        if (tp < tq) {
          const int b = tp & 1;
          if (mbar_test_wait(p_full(b), (tp >> 1) & 1) && mbar_test_wait(v_full, tp & 1)) {
            ok = issue_pv(tp);  // its waits succeed at once
            if (!ok) break;
            ++tp;
            progress = true;
          }
        }
        if (have_q && tq <= tp + 1) {
          const int b = tq & 1;
          if (mbar_test_wait(q_rot(b), (tq >> 1) & 1) && mbar_test_wait(k_full, tq & 1) &&
              (tq < 2 || mbar_test_wait(o_empty(b), ((tq >> 1) - 1) & 1))) {
            issue_qk(tq);
            ++tq;
            TileInfo T;
            have_q = locate<0>(p, S, blockIdx.x + tq * gridDim.x, T);
            progress = true;
          }
        }
        if (progress) {
          t_last = global_timer_ns();
        } else if (!*abort_flag && global_timer_ns() - t_last <= p.wait_ns) {
          __nanosleep(32);  // yield the issue slots this sub-partition shares with softmax warps
        } else if (*abort_flag) {
          ok = false;
          break;
        } else if (global_timer_ns() - t_last > p.wait_ns) {
          *abort_flag = 1;
          atomicOr(status, MIMO_STATUS_TIMEOUT);
          ok = false;
          break;
        }
      }
      if (!ok) {
        int dummy = 0;
        tc_commit(drain);
        mbar_wait(drain, 0, &dummy, nullptr, 0, 50000000ull);
      }
    }
    __syncwarp();
  } else if (warp >= 10) {
    // ------------------------------------------------------------ Q RoPE (warps 10, 11)
    // Dims 0..63 of the tile's 128 rows are rotated in place (128-byte swizzled rows)
    // to fp16 with the (cos, sin) rows the producer loaded next to the Q tile.
    const int lt = threadIdx.x - 320;  // 0..63
    bool ok = true;
    for (int mt = 0, w = blockIdx.x; ok; ++mt, w += gridDim.x) {
      TileInfo T;
      if (!locate<0>(p, S, w, T)) break;
      const int b = mt & 1;
      if (!(ok = mbar_wait(q_full(b), (mt >> 1) & 1, abort_flag, status, MIMO_STATUS_TIMEOUT, p.wait_ns))) break;
      const float4* cs = reinterpret_cast<const float4*>(smem + Ly::kOffCS + b * Ly::kCSStage);
      uint8_t* qs = smem + Ly::kOffQ + b * Ly::kQStage;
      float amax = 0.f;  // every row holds a real query (or TMA zero fill past total_q)
      // work item k: head h = k & 7, chunk pair u = (k >> 3) & 3, position r = k >> 5 (row 8r + h):
      // the 8 lanes of a shared-memory phase hit 8 distinct swizzled 16-byte groups of Q and
      // read one broadcast (cos, sin) address.
#pragma unroll 2
      for (int i = 0; i < 128 * 4 / 64; ++i) {
        const int k = lt + 64 * i;
        const int m = ((k >> 5) << 3) + (k & 7), u = (k >> 3) & 3, sw = m & 7;
        uint8_t* row = qs + m * 128;
        uint4* plo = reinterpret_cast<uint4*>(row + ((u ^ sw) << 4));
        uint4* phi = reinterpret_cast<uint4*>(row + (((u + 4) ^ sw) << 4));
        uint4 lo = *plo, hi = *phi;
        // (cos, sin) of frequencies 8u..8u+7 at the row's position: 4 x float4
        rope_chunk_pair_cs4(lo, hi, cs + (m / G) * 16 + 4 * u, amax);
        *plo = lo;
        *phi = hi;
      }
      if (amax > kF16Max) atomicOr(status, MIMO_STATUS_RANGE);
      fence_proxy_async_smem();
      mbar_arrive(q_rot(b));
    }
  } else {
    // ------------------------------------------------------------ two softmax warpgroups
    const int wg = (warp - 2) >> 2;        // 0: warps 2..5, 1: warps 6..9
    const int quad = warp & 3;
    const int m = quad * 32 + lane;        // TMEM lane = M row
    const int r = m / G, hq = m % G;
    const uint32_t t_lane = tmem + (uint32_t(quad * 32) << 16) + wg * kSwaRegion;
    const float c_log2 = p.scale_log2;
    auto wait_w = [&](uint32_t bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, status, MIMO_STATUS_TIMEOUT, p.wait_ns));
    };
    for (int mt = wg, w = blockIdx.x + wg * gridDim.x;; mt += 2, w += 2 * gridDim.x) {
      TileInfo T;
      if (!locate<0>(p, S, w, T)) break;
      const int b = wg;  // == mt & 1
      const uint32_t ph = (mt >> 1) & 1;
      // ---- softmax over the 144-key tile, two passes of 72 columns
      const bool row_valid = r < T.rows_valid;
      const int qp = T.qpos0 + r;
      const int head = T.g * G + hq;
      const int kt0 = T.qpos0 - 128;
      const int vis_hi = row_valid ? qp : -0x40000000;
      const int vis_lo = max(T.key_lo, qp - p.window + 1);
      const int ca = vis_lo - kt0, ce = vis_hi - kt0;  // visible columns [ca, ce]
      if (!wait_w(s_full(b), ph)) break;
      tc_fence_after();
      // Columns 16..127 of the tile are visible to all 16 positions whenever the whole
      // window exists (ca <= 16, ce >= 127 for every row): only the 16 edge columns
      // on each side need the per-element mask then.
      const bool band = __all_sync(0xffffffffu, ca <= 16 && ce >= 127);
      const float sink = sink_l2[head];
      float m_use, la[4];
      if (band) {
        // Columns 16..127 are visible to every row; the edge columns are the first half of
        // chunk 0 and all of chunk 4 (chunks of 32 columns, the last one 16).  One pass over
        // S: chunk 4 (keys q0 .. q0+15) holds every row's own key, so its visible maximum
        // (with the sink) is the reference m_use of the exponentials of all chunks; the
        // softmax needs no exact row maximum, only no overflow, and the LSE is
        // m_use + log2(sum).  A chunk whose sum overflows 2^64 (a logit far above the
        // reference) raises m_use to its maximum and rescales the P already written.
        // TMEM loads run one chunk ahead (two register buffers).
        uint32_t buf[2][32];
        auto ld = [&](int h, uint32_t* d) {
          if (h < 4) tmem_ld32(t_lane + 32 * h, d);
          else tmem_ld16(t_lane + 128, d);
        };
        auto edge_col = [&](int h, int c) { return (h == 0 && c < 16) || h == 4; };
        auto vis_col = [&](int h, int c) {
          const int cc = 32 * h + c;
          return !edge_col(h, c) || (cc >= ca && cc <= ce);
        };
        auto chunk_max = [&](const uint32_t* sr, int h) {
          float mx = -INFINITY;
#pragma unroll
          for (int c = 0; c < (h < 4 ? 32 : 16); ++c)
            if (vis_col(h, c)) mx = fmaxf(mx, __uint_as_float(sr[c]));
          return mx;
        };
        ld(4, buf[0]);
        ld(0, buf[1]);
        tmem_wait_ld_r16(buf[0]);
        {
          const float m_row = fmaxf(sink, chunk_max(buf[0], 4) * c_log2);
          m_use = m_row == -INFINITY ? 0.f : m_row;
        }
        const uint64_t cl2 = pack_f32x2(c_log2, c_log2);
        uint64_t la2 = pack_f32x2(p.sink ? ex2(sink - m_use) : 0.f, 0.f);
        // exponentials of one chunk into packed bf16 words; returns the chunk's sum
        auto exp_chunk = [&](const uint32_t* sr, int h, uint32_t* pk) {
          const uint64_t nm2 = pack_f32x2(-m_use, -m_use);
          uint64_t sum2 = pack_f32x2(0.f, 0.f);
#pragma unroll
          for (int c = 0; c < (h < 4 ? 32 : 16); c += 2) {
            const uint64_t t = fma_f32x2(pack_f32x2(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])), cl2, nm2);
            float p0 = ex2(lo_f32(t)), p1 = ex2(hi_f32(t));
            if (edge_col(h, c)) {
              p0 = vis_col(h, c) ? p0 : 0.f;
              p1 = vis_col(h, c + 1) ? p1 : 0.f;
            }
            sum2 = add_f32x2(sum2, pack_f32x2(p0, p1));
            pk[c / 2] = pack_bf16x2(p0, p1);
          }
          return lo_f32(sum2) + hi_f32(sum2);
        };
        // rare: rows whose chunk sum overflowed take the chunk's maximum as the new
        // reference; P columns [0, written) in TMEM, the held chunk-4 words and the running
        // sum are scaled down to it (warp-uniform loop: TMEM access is warp-collective)
        uint32_t pk4[8];
        auto raise_ref = [&](bool over, const uint32_t* sr, int h, int written) {
          tmem_wait_st();
          float f = 1.f;
          if (over) {
            const float m_new = fmaxf(m_use, chunk_max(sr, h) * c_log2);
            f = ex2(m_use - m_new);
            m_use = m_new;
          }
          const uint64_t f2 = pack_f32x2(f, f);
          la2 = mul_f32x2(la2, f2);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const uint64_t t = mul_f32x2(pack_f32x2(lo_bf16(pk4[i]), hi_bf16(pk4[i])), f2);
            pk4[i] = pack_bf16x2(lo_f32(t), hi_f32(t));
          }
#pragma unroll 1
          for (int c0 = 0; c0 < written; c0 += 8) {
            uint32_t w[8];
            tmem_ld8(t_lane + c0, w);
            tmem_wait_ld_r8(w);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const uint64_t t = mul_f32x2(pack_f32x2(lo_bf16(w[i]), hi_bf16(w[i])), f2);
              w[i] = pack_bf16x2(lo_f32(t), hi_f32(t));
            }
            tmem_st8(t_lane + c0, w);
          }
          tmem_wait_st();
        };
        constexpr float kOver = 18446744073709551616.f;  // 2^64
        {
          float sum = exp_chunk(buf[0], 4, pk4);
          if (__any_sync(0xffffffffu, !(sum <= kOver))) {
            raise_ref(!(sum <= kOver), buf[0], 4, 0);
            sum = exp_chunk(buf[0], 4, pk4);
          }
          la2 = add_f32x2(la2, pack_f32x2(sum, 0.f));
        }
        tmem_wait_ld_r32(buf[1]);
        {  // chunk 0: columns 0..15 are edge columns
          uint32_t pk[16];
          float sum = exp_chunk(buf[1], 0, pk);
          if (__any_sync(0xffffffffu, !(sum <= kOver))) {
            raise_ref(!(sum <= kOver), buf[1], 0, 0);
            sum = exp_chunk(buf[1], 0, pk);
          }
          tmem_st8(t_lane, pk);
          tmem_st8(t_lane + 8, pk + 8);
          la2 = add_f32x2(la2, pack_f32x2(sum, 0.f));
        }
        // chunks 1..3: every column visible; one copy of the code for the three
        auto exp_mid = [&](const uint32_t* sr, uint32_t* pk) {
          const uint64_t nm2 = pack_f32x2(-m_use, -m_use);
          uint64_t sum2 = pack_f32x2(0.f, 0.f);
#pragma unroll
          for (int c = 0; c < 32; c += 2) {
            const uint64_t t = fma_f32x2(pack_f32x2(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])), cl2, nm2);
            const float p0 = ex2(lo_f32(t)), p1 = ex2(hi_f32(t));
            sum2 = add_f32x2(sum2, pack_f32x2(p0, p1));
            pk[c / 2] = pack_bf16x2(p0, p1);
          }
          return lo_f32(sum2) + hi_f32(sum2);
        };
#pragma unroll 1
        for (int h = 1; h < 4; ++h) {
          tmem_ld32(t_lane + 32 * h, buf[0]);
          tmem_wait_ld_r32(buf[0]);
          uint32_t pk[16];
          float sum = exp_mid(buf[0], pk);
          if (__any_sync(0xffffffffu, !(sum <= kOver))) {
            raise_ref(!(sum <= kOver), buf[0], h, 16 * h);
            sum = exp_mid(buf[0], pk);
          }
          tmem_st8(t_lane + 16 * h, pk);
          tmem_st8(t_lane + 16 * h + 8, pk + 8);
          la2 = add_f32x2(la2, pack_f32x2(sum, 0.f));
        }
        tmem_st8(t_lane + 64, pk4);
        la[0] = lo_f32(la2);
        la[1] = hi_f32(la2);
        la[2] = la[3] = 0.f;
      } else {
        float mxa[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll 1
        for (int h = 0; h < 3; ++h) {
          uint32_t sr[CH];
          tmem_ld32(t_lane + h * CH, sr);
          tmem_ld16(t_lane + h * CH + 32, sr + 32);
          tmem_wait_ld_r32(sr);
          tmem_wait_ld_r16(sr + 32);
#pragma unroll
          for (int c = 0; c < CH; ++c) {
            const int cc = h * CH + c;
            if (cc >= ca && cc <= ce) mxa[c & 3] = fmaxf(mxa[c & 3], __uint_as_float(sr[c]));
          }
        }
        const float mx = fmaxf(fmaxf(mxa[0], mxa[1]), fmaxf(mxa[2], mxa[3]));
        const float m_row = fmaxf(sink, mx * c_log2);
        m_use = m_row == -INFINITY ? 0.f : m_row;
        la[0] = p.sink ? ex2(sink - m_use) : 0.f;
        la[1] = la[2] = la[3] = 0.f;
#pragma unroll 1
        for (int h = 0; h < 3; ++h) {
          uint32_t sr[CH];
          tmem_ld32(t_lane + h * CH, sr);
          tmem_ld16(t_lane + h * CH + 32, sr + 32);
          tmem_wait_ld_r32(sr);
          tmem_wait_ld_r16(sr + 32);
          uint32_t pk[CH / 2];
#pragma unroll
          for (int c = 0; c < CH; c += 2) {
            const int cc = h * CH + c;
            float p0 = ex2(fmaf(__uint_as_float(sr[c]), c_log2, -m_use));
            float p1 = ex2(fmaf(__uint_as_float(sr[c + 1]), c_log2, -m_use));
            p0 = (cc >= ca && cc <= ce) ? p0 : 0.f;
            p1 = (cc + 1 >= ca && cc + 1 <= ce) ? p1 : 0.f;
            la[(c >> 1) & 3] += p0 + p1;
            pk[c / 2] = pack_bf16x2(p0, p1);
          }
          tmem_st16(t_lane + h * (CH / 2), pk);
          tmem_st8(t_lane + h * (CH / 2) + 16, pk + 16);
        }
      }
      const float l_row = (la[0] + la[1]) + (la[2] + la[3]);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(p_full(b));
      // ---- epilogue: O * v_scale / l -> bf16, LSE
      if (!wait_w(pv_done(b), ph)) break;
      tc_fence_after();
      const float sc = p.v_scale / l_row;
      {
        // O rows go out through a per-warp staging buffer, 32 columns at a time: each
        // thread writes its row's 64 bytes (16-byte units XOR-swizzled by row pair), then
        // a store instruction writes 64 contiguous bytes of each of 8 rows (one position,
        // the 8 heads) instead of 16 bytes of each of 32 rows.
        uint8_t* stage = smem + Ly::kOffStage + (warp - 2) * Ly::kStageBytes;
        const uint64_t sc2 = pack_f32x2(sc, sc);
        uint32_t oa[32];
        auto store_chunk = [&](uint32_t* o, int c) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const uint64_t t = mul_f32x2(pack_f32x2(__uint_as_float(o[2 * i]), __uint_as_float(o[2 * i + 1])), sc2);
            o[i] = pack_bf16x2(lo_f32(t), hi_f32(t));
          }
#pragma unroll
          for (int u = 0; u < 4; ++u)
            *reinterpret_cast<uint4*>(stage + lane * 64 + ((u ^ ((lane >> 1) & 3)) << 4)) =
                make_uint4(o[4 * u], o[4 * u + 1], o[4 * u + 2], o[4 * u + 3]);
          __syncwarp();
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int rho = 8 * k + (lane >> 2), u = lane & 3;  // warp row (position quad*4 + k, head rho % 8)
            const uint4 v = *reinterpret_cast<const uint4*>(stage + rho * 64 + ((u ^ ((rho >> 1) & 3)) << 4));
            if (quad * 4 + k < T.rows_valid)
              *reinterpret_cast<uint4*>(p.out + (long(T.q_row0 + quad * 4 + k) * kHq + T.g * G + (lane >> 2)) * kDv +
                                        c + 8 * u) = v;
          }
          __syncwarp();
        };
#pragma unroll 1
        for (int c = 0; c < 128; c += 32) {
          tmem_ld32(t_lane + kSwaColO + c, oa);
          tmem_wait_ld_r32(oa);
          store_chunk(oa, c);
        }
      }
      if (row_valid && p.lse) p.lse[long(T.q_row0 + r) * kHq + head] = (m_use + __log2f(l_row)) * kLn2;
      tc_fence_before();
      mbar_arrive(o_empty(b));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------- key pre-pass
// Largest s in [0, n) with off(s) <= x (off non-decreasing), for a whole warp that passes
// the same x: up to 32 sequences with one load per lane and a ballot (one memory round
// trip, where a bisection takes log2 n dependent ones), else by bisection.
template <typename F>
__device__ __forceinline__ int warp_find_seq(int n, long x, F off) {
  if (n <= 32) {
    const int lane = threadIdx.x & 31;
    const unsigned m = __ballot_sync(0xffffffffu, lane < n && off(lane) <= x);
    return m ? 31 - __clz(m) : 0;
  }
  int lo = 0, hi = n;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (off(mid) <= x) lo = mid; else hi = mid;
  }
  return lo;
}

// Position of query row `row` (warp-collective): the queries of a sequence are the last
// q_len of its ctx = cached + new keys.
__device__ __forceinline__ int query_position(const RopeKParams& p, long row) {
  const int lo = warp_find_seq(p.num_seqs, row, [&](int i) { return long(p.cu_q[i]); });
  const int qlen = p.cu_q[lo + 1] - p.cu_q[lo];
  const int ctx = (p.cache_lens ? p.cache_lens[lo] : 0) + (p.cu_k[lo + 1] - p.cu_k[lo]);
  return ctx - qlen + int(row - p.cu_q[lo]);
}

// contig: one warp per key row.  Lane j computes frequency j's (cos, sin) at the row's
// position once; lane l rotates chunk pair (head l / 4, u = l % 4) of dims 0..63 with the
// pairs of frequencies 8u..8u+7 taken from the lanes that hold them, and writes it (fp16)
// into ws_k.  The loads are issued before the trig so that their latency overlaps it.  For
// query rows (when cs_q is set) the same warp writes the row's (cos, sin) at the query's
// position, reusing the key's when the two positions agree (prefill without a cache).  One
// sine / cosine per lane keeps the latency of a short call low (eight per thread before).
template <int HKV>
__global__ void __launch_bounds__(256) rope_k_contig_kernel(const RopeKParams p) {
  static_assert(HKV * 4 <= 32, "one rotated chunk pair per lane");
  pdl_launch_dependents();
  const long row = (long(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const bool key_row = row < p.total_k;
  const bool q_row = p.cs_q && row < p.total_q;
  if (!key_row && !q_row) return;  // warp-uniform: one row per warp
  int pos_k = 0;
  float c_j = 0.f, s_j = 0.f;
  if (key_row) {
    const int g = lane >> 2, u = lane & 3;
    const bool act = g < HKV;
    uint4 a = make_uint4(0, 0, 0, 0), b = a;
    const uint4* src = reinterpret_cast<const uint4*>(p.k + (row * HKV + g) * kDqk) + u;
    if (act) {
      a = __ldg(src);
      b = __ldg(src + 4);
    }
    // s with cu_k[s] <= row < cu_k[s+1]
    const int lo = warp_find_seq(p.num_seqs, row, [&](int i) { return long(p.cu_k[i]); });
    pos_k = (p.cache_lens ? p.cache_lens[lo] : 0) + int(row - p.cu_k[lo]);
    rope_cos_sin(pos_k, p.rope.inv_freq[lane], &c_j, &s_j);
    float2 cs[8];
#pragma unroll
    for (int f = 0; f < 8; ++f) {
      cs[f].x = __shfl_sync(0xffffffffu, c_j, 8 * u + f);
      cs[f].y = __shfl_sync(0xffffffffu, s_j, 8 * u + f);
    }
    if (act) {
      float amax = 0.f;
      rope_chunk_pair_cs(a, b, cs, amax);
      if (amax > kF16Max) atomicOr(p.status, MIMO_STATUS_RANGE);
      uint4* dst = reinterpret_cast<uint4*>(p.ws_k + (row * HKV + g) * kRope) + u;
      dst[0] = a;
      dst[4] = b;
    }
  }
  if (q_row) {
    const int pos_q = query_position(p, row);
    if (!key_row || pos_q != pos_k) rope_cos_sin(pos_q, p.rope.inv_freq[lane], &c_j, &s_j);
    p.cs_q[row * kHalf + lane] = make_float2(c_j, s_j);
  }
}

// ext: one warp per row e of [128-slot ring halo | new keys] of each sequence.  It writes
// the whole key of all HKV heads (dims 0..63 rotated fp16, 64..191 bf16) and the value:
// halo rows are copied from the ring (which holds that format; zeros before the sequence
// start), new rows are rotated from k / v.  Lane j computes frequency j's (cos, sin)
// once; lane l rotates chunk pair (head l / 4, u = l % 4) with the pairs of frequencies
// 8u..8u+7 taken from the lanes that hold them.  The same warp also fills query row e's
// cos/sin row when cs_q is set.
template <int HKV>
__global__ void __launch_bounds__(256) rope_k_ext_kernel(const RopeKParams p) {
  static_assert(HKV * 4 <= 32, "one rotated chunk pair per lane");
  constexpr int kKRow = HKV * kDqk / 8;  // uint4 of one position's keys (all heads)
  constexpr int kVRow = HKV * kDv / 8;
  pdl_launch_dependents();
  const long wid = (long(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const long rows = long(p.total_k) + 128L * p.num_seqs;
  const bool key_row = wid < rows;
  const bool q_row = p.cs_q && wid < p.total_q;
  if (!key_row && !q_row) return;
  int pos_k = 0;
  bool have_cs = false;  // c_j, s_j hold frequency `lane` at pos_k (warp-uniform)
  float c_j = 0.f, s_j = 0.f;
  if (key_row) {
    const int e = int(wid);
    // the sequence whose ext rows (its 128 halo rows, then its new rows) hold row e
    const int lo = warp_find_seq(p.num_seqs, e, [&](int i) { return long(p.cu_k[i]) + 128L * i; });
    const int s = lo, i = e - (p.cu_k[s] + 128 * s);
    const int clen = p.cache_lens ? p.cache_lens[s] : 0;
    uint4* kd = reinterpret_cast<uint4*>(p.ws_k + long(e) * HKV * kDqk);
    uint4* vd = reinterpret_cast<uint4*>(p.ws_v + long(e) * HKV * kDv);
    if (i < 128) {
      const int pos = clen - 128 + i;
      if (pos < 0) {
        for (int t = lane; t < kKRow; t += 32) kd[t] = make_uint4(0, 0, 0, 0);
        for (int t = lane; t < kVRow; t += 32) vd[t] = make_uint4(0, 0, 0, 0);
      } else {
        const long entry = long(s) * p.ring_slots + (pos % p.ring_slots);
        const uint4* ks = reinterpret_cast<const uint4*>(p.ring_k + entry * HKV * kDqk);
        const uint4* vs = reinterpret_cast<const uint4*>(p.ring_v + entry * HKV * kDv);
        uint4 kr[(kKRow + 31) / 32], vr[(kVRow + 31) / 32];
#pragma unroll
        for (int t = 0; t < (kKRow + 31) / 32; ++t)
          if (lane + 32 * t < kKRow) kr[t] = __ldg(ks + lane + 32 * t);
#pragma unroll
        for (int t = 0; t < (kVRow + 31) / 32; ++t)
          if (lane + 32 * t < kVRow) vr[t] = __ldg(vs + lane + 32 * t);
#pragma unroll
        for (int t = 0; t < (kKRow + 31) / 32; ++t)
          if (lane + 32 * t < kKRow) kd[lane + 32 * t] = kr[t];
#pragma unroll
        for (int t = 0; t < (kVRow + 31) / 32; ++t)
          if (lane + 32 * t < kVRow) vd[lane + 32 * t] = vr[t];
      }
    } else {
      const long row = p.cu_k[s] + (i - 128);
      pos_k = clen + (i - 128);
      // every new row: its rotated dims 0..63 into ws_rot (the tiles whose window starts inside
      // the chunk read those with k and v); the first kExtFullRows rows also whole into the
      // ext copy, for the tiles whose window reaches back into the halo
      const bool full_row = i - 128 < kExtFullRows;  // warp-uniform
      const uint4* ks = reinterpret_cast<const uint4*>(p.k + row * HKV * kDqk);
      const uint4* vs = reinterpret_cast<const uint4*>(p.v + row * HKV * kDv);
      // rotated pair of this lane, the plain key chunks (dims 64..191) and the value
      constexpr int kPlain = HKV * 16 / 32, kVal = kVRow / 32;
      const int pg = lane >> 2, pu = lane & 3;
      const bool has_pair = pg < HKV;
      uint4 ra, rb, kp[kPlain], vv[kVal];
      if (has_pair) {
        ra = __ldg(ks + pg * (kDqk / 8) + pu);
        rb = __ldg(ks + pg * (kDqk / 8) + pu + 4);
      }
      if (full_row) {
#pragma unroll
        for (int t = 0; t < kPlain; ++t) {
          const int c = lane + 32 * t;
          kp[t] = __ldg(ks + (c >> 4) * (kDqk / 8) + 8 + (c & 15));
        }
#pragma unroll
        for (int t = 0; t < kVal; ++t) vv[t] = __ldg(vs + lane + 32 * t);
      }
      rope_cos_sin(pos_k, p.rope.inv_freq[lane], &c_j, &s_j);
      have_cs = true;
      float2 cs[8];
#pragma unroll
      for (int f = 0; f < 8; ++f) {
        cs[f].x = __shfl_sync(0xffffffffu, c_j, 8 * pu + f);
        cs[f].y = __shfl_sync(0xffffffffu, s_j, 8 * pu + f);
      }
      if (has_pair) {
        float amax = 0.f;
        rope_chunk_pair_cs(ra, rb, cs, amax);
        if (amax > kF16Max) atomicOr(p.status, MIMO_STATUS_RANGE);
        uint4* rot = reinterpret_cast<uint4*>(p.ws_rot + (row * HKV + pg) * kRope) + pu;
        rot[0] = ra;
        rot[4] = rb;
        if (full_row) {
          kd[pg * (kDqk / 8) + pu] = ra;
          kd[pg * (kDqk / 8) + pu + 4] = rb;
        }
      }
      if (full_row) {
#pragma unroll
        for (int t = 0; t < kPlain; ++t) {
          const int c = lane + 32 * t;
          kd[(c >> 4) * (kDqk / 8) + 8 + (c & 15)] = kp[t];
        }
#pragma unroll
        for (int t = 0; t < kVal; ++t) vd[lane + 32 * t] = vv[t];
      }
    }
  }
  if (q_row) {
    const int pos_q = query_position(p, wid);
    if (!have_cs || pos_q != pos_k) rope_cos_sin(pos_q, p.rope.inv_freq[lane], &c_j, &s_j);
    p.cs_q[wid * kHalf + lane] = make_float2(c_j, s_j);
  }
}

cudaError_t launch_rope_k(const RopeKParams& p, cudaStream_t s) {
  if (p.hkv != 4 && p.hkv != 8) return cudaErrorInvalidValue;
  const long qrows = p.cs_q ? long(p.total_q) : 0;
  if (p.mode == kModeContig) {
    const long rows = long(p.total_k) > qrows ? long(p.total_k) : qrows;
    const long blocks = (rows * 32 + 255) / 256;
    if (blocks == 0) return cudaSuccess;
    if (p.hkv == 8) rope_k_contig_kernel<8><<<unsigned(blocks), 256, 0, s>>>(p);
    else rope_k_contig_kernel<4><<<unsigned(blocks), 256, 0, s>>>(p);
  } else {
    const long ext = long(p.total_k) + 128L * p.num_seqs;
    const long rows = ext > qrows ? ext : qrows;
    const long blocks = (rows * 32 + 255) / 256;
    if (blocks == 0) return cudaSuccess;
    if (p.hkv == 8) rope_k_ext_kernel<8><<<unsigned(blocks), 256, 0, s>>>(p);
    else rope_k_ext_kernel<4><<<unsigned(blocks), 256, 0, s>>>(p);
  }
  return cudaGetLastError();
}

int prefill_rows_per_tile(int kind) { return kind == 0 ? Cfg<0>::R : Cfg<1>::R; }  // query rows of one TMA box
int prefill_key_tile(int kind) { return kind == 0 ? Cfg<0>::BN : Cfg<1>::BN; }

cudaError_t launch_prefill(const PrefillParams& p, int kind, int grid, cudaStream_t s, bool pdl) {
  if (grid <= 0) return cudaSuccess;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(grid));
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  if (kind == 0) {
    cudaError_t e = cudaFuncSetAttribute(prefill_swa_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         SwaLayout::kAlloc);
    if (e != cudaSuccess) return e;
    cfg.blockDim = dim3(kSwaThreads);
    cfg.dynamicSmemBytes = SwaLayout::kAlloc;
    return cudaLaunchKernelEx(&cfg, prefill_swa_kernel, p);
  }
  auto* fn = p.split_tiles > 0 ? prefill_kernel<1, true> : prefill_kernel<1, false>;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, Layout<1>::kAlloc);
  if (e != cudaSuccess) return e;
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = Layout<1>::kAlloc;
  return cudaLaunchKernelEx(&cfg, fn, p);
}

}  // namespace mimo
