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
struct Cfg<0> {  // sliding window
  static constexpr int G = 8, R = 16, BN = 144, NQ = 2, NK = 1, NV = 1;
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
  static constexpr int kOffCS = kOffSink + 64 * 4;                    // float2 [R][32] cos/sin of a tile
  static constexpr int kBytes = kOffCS + C::R * 32 * 8;
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
      const int q0 = p.cu_q[s], ql = p.cu_q[s + 1] - q0;
      n = (ql + R - 1) / R;
      S.q0[s] = q0;
      S.qlen[s] = ql;
      S.clen[s] = p.cache_lens ? p.cache_lens[s] : 0;
      S.k0[s] = p.cu_k ? p.cu_k[s] : 0;
      S.klen[s] = p.cu_k ? p.cu_k[s + 1] - p.cu_k[s] : 0;
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
// global attention.
template <int KIND>
__device__ __forceinline__ bool locate(const PrefillParams& p, const SeqTable& S, int w, TileInfo& T) {
  constexpr int R = Cfg<KIND>::R;
  const int tt = w / p.hkv;
  if (tt >= S.tile_start[p.num_seqs]) return false;
  int lo = 0, hi = p.num_seqs;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (S.tile_start[mid] <= tt) lo = mid; else hi = mid;
  }
  T.s = lo;
  T.ntiles = S.tile_start[lo + 1] - S.tile_start[lo];
  int t = tt - S.tile_start[lo];
  if (KIND == 1) t = T.ntiles - 1 - t;
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
  }
}
template <int KIND>
__device__ __forceinline__ int key_tile_start(const TileInfo& T, int j) {
  return KIND == 0 ? T.qpos0 - 128 : j * 128;
}

}  // namespace

template <int KIND>
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
      int mt = 0, jj = 0;
      bool ok = true;
      for (int w = blockIdx.x; ok; w += gridDim.x) {
        TileInfo T;
        if (!locate<KIND>(p, S, w, T)) break;
        if (lane == 0) {
          const int qs = mt % NQ;
          if (mt >= NQ) ok = mbar_wait(q_empty(qs), ((mt / NQ) - 1) & 1, abort_flag, status, MIMO_STATUS_TIMEOUT);
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
              if (jj >= NK) ok = mbar_wait(k_empty(ks), ((jj / NK) - 1) & 1, abort_flag, status, MIMO_STATUS_TIMEOUT);
              if (!ok) break;
              const uint32_t kdst = sbase + Ly::kOffK + ks * Ly::kKStage;
              mbar_expect_tx(k_full(ks), Ly::kKStage);
              tma_load_3d(kdst, &p.tm_k0, k_full(ks), 0, T.g, row);
              tma_load_3d(kdst + Ly::kKChunk, &p.tm_k12, k_full(ks), 64, T.g, row);
              tma_load_3d(kdst + 2 * Ly::kKChunk, &p.tm_k12, k_full(ks), 128, T.g, row);
            } else {
              const int vs = jj % NV;
              if (jj >= NV) ok = mbar_wait(v_empty(vs), ((jj / NV) - 1) & 1, abort_flag, status, MIMO_STATUS_TIMEOUT);
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
        if (!mbar_wait(p_full(b), (jp >> 1) & 1, abort_flag, status, MIMO_STATUS_TIMEOUT)) return false;
        const int vs = jp % NV;
        if (!mbar_wait(v_full(vs), (jp / NV) & 1, abort_flag, status, MIMO_STATUS_TIMEOUT)) return false;
        if (first && mtp > 0 && !mbar_wait(o_empty, (mtp - 1) & 1, abort_flag, status, MIMO_STATUS_TIMEOUT))
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
        if (!(ok = mbar_wait(q_rot(qs), (mt / NQ) & 1, abort_flag, status, MIMO_STATUS_TIMEOUT))) break;
        tc_fence_after();
        int j_lo, nkv;
        key_tiles<KIND>(p, T, &j_lo, &nkv);
        const uint32_t qbase = sbase + Ly::kOffQ + qs * Ly::kQStage;
        for (int j = 0; j < nkv; ++j) {
          const int ks = jj % NK;
          if (!(ok = mbar_wait(k_full(ks), (jj / NK) & 1, abort_flag, status, MIMO_STATUS_TIMEOUT))) break;
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
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, status, MIMO_STATUS_TIMEOUT));
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
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        uint4* plo = reinterpret_cast<uint4*>(row + ((u ^ sw) << 4));
        uint4* phi = reinterpret_cast<uint4*>(row + (((u + 4) ^ sw) << 4));
        uint4 lo = *plo, hi = *phi;
        rope_chunk_pair_cs(lo, hi, csr + 8 * u);
        *plo = lo;
        *phi = hi;
      }
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
      float m_run = sink_l2[head];
      float l_run = p.sink ? 1.f : 0.f;
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
        tmem_wait_ld();
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
        if (j > 0 && !(ok = wait_w(pv_done, (jj - 1) & 1))) break;
        const float m_new = fmaxf(m_run, mt_l2);
        float alpha = 1.f;
        const bool resc = m_new > m_run + 8.f;
        if (resc) {
          alpha = ex2(m_run - m_new);
          m_run = m_new;
        }
        if (__any_sync(0xffffffffu, resc && j > 0)) {
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < 128; c += 32) {
            uint32_t o[32];
            tmem_ld32(t_lane + kColO + c, o);
            tmem_wait_ld();
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
      // ---- epilogue
      if (!(ok = wait_w(pv_done, (jj - 1) & 1))) break;
      tc_fence_after();
      const float sc = p.v_scale / l_run;
      uint16_t* orow = p.out + (long(T.q_row0 + r) * kHq + head) * kDv;
#pragma unroll
      for (int c = 0; c < 128; c += 32) {
        uint32_t o[32];
        tmem_ld32(t_lane + kColO + c, o);
        tmem_wait_ld();
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

// ---------------------------------------------------------------- key pre-pass
// contig: 4 lanes per (row, kv head) write rotated dims 0..63 (fp16) into ws_k.
// ext: one warp per (ext row, kv head) writes the full rotated key (dims 0..63
//      fp16, 64..191 bf16) and the value: halo rows copied from the ring (which
//      stores the same format), new rows rotated from k / v.
__global__ void __launch_bounds__(256) rope_k_kernel(const RopeKParams p) {
  const long gt = long(blockIdx.x) * blockDim.x + threadIdx.x;
  if (p.mode == kModeContig) {
    const long item = gt >> 2;
    const int u = int(gt & 3);
    if (item >= long(p.total_k) * p.hkv) return;
    const int row = int(item / p.hkv), g = int(item % p.hkv);
    int lo = 0, hi = p.num_seqs;  // find s with cu_k[s] <= row < cu_k[s+1]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (p.cu_k[mid] <= row) lo = mid; else hi = mid;
    }
    const int pos = (p.cache_lens ? p.cache_lens[lo] : 0) + (row - p.cu_k[lo]);
    const uint4* src = reinterpret_cast<const uint4*>(p.k + (long(row) * p.hkv + g) * kDqk);
    uint4 a = __ldg(src + u), b = __ldg(src + u + 4);
    rope_chunk_pair(a, b, u, pos, p.rope);
    uint4* dst = reinterpret_cast<uint4*>(p.ws_k + (long(row) * p.hkv + g) * kRope);
    dst[u] = a;
    dst[u + 4] = b;
    return;
  }
  const long wid = gt >> 5;
  const int lane = int(gt & 31);
  const long rows = long(p.total_k) + 128L * p.num_seqs;
  if (wid >= rows * p.hkv) return;
  const int e = int(wid / p.hkv), g = int(wid % p.hkv);
  int lo = 0, hi = p.num_seqs;  // ext start of s: cu_k[s] + 128 s
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (p.cu_k[mid] + 128 * mid <= e) lo = mid; else hi = mid;
  }
  const int s = lo, i = e - (p.cu_k[s] + 128 * s);
  const int clen = p.cache_lens ? p.cache_lens[s] : 0;
  uint4* kd = reinterpret_cast<uint4*>(p.ws_k + (long(e) * p.hkv + g) * kDqk);
  uint4* vd = reinterpret_cast<uint4*>(p.ws_v + (long(e) * p.hkv + g) * kDv);
  if (i < 128) {
    const int pos = clen - 128 + i;
    if (pos < 0) {
      if (lane < 24) kd[lane] = make_uint4(0, 0, 0, 0);
      if (lane < 16) vd[lane] = make_uint4(0, 0, 0, 0);
      return;
    }
    const long entry = long(s) * kPage + (pos % kPage);
    const uint4* ks = reinterpret_cast<const uint4*>(p.ring_k + (entry * p.hkv + g) * kDqk);
    const uint4* vs = reinterpret_cast<const uint4*>(p.ring_v + (entry * p.hkv + g) * kDv);
    if (lane < 24) kd[lane] = __ldg(ks + lane);
    if (lane < 16) vd[lane] = __ldg(vs + lane);
    return;
  }
  const int row = p.cu_k[s] + (i - 128);
  const int pos = clen + (i - 128);
  const uint4* ks = reinterpret_cast<const uint4*>(p.k + (long(row) * p.hkv + g) * kDqk);
  if (lane < 4) {
    uint4 a = __ldg(ks + lane), b = __ldg(ks + lane + 4);
    rope_chunk_pair(a, b, lane, pos, p.rope);
    kd[lane] = a;
    kd[lane + 4] = b;
  } else if (lane >= 8 && lane < 24) {
    kd[lane] = __ldg(ks + lane);
  }
  if (lane < 16) vd[lane] = __ldg(reinterpret_cast<const uint4*>(p.v + (long(row) * p.hkv + g) * kDv) + lane);
}

cudaError_t launch_rope_k(const RopeKParams& p, cudaStream_t s) {
  long threads;
  if (p.mode == kModeContig) threads = long(p.total_k) * p.hkv * 4;
  else threads = (long(p.total_k) + 128L * p.num_seqs) * p.hkv * 32;
  if (threads == 0) return cudaSuccess;
  rope_k_kernel<<<unsigned((threads + 255) / 256), 256, 0, s>>>(p);
  return cudaGetLastError();
}

int prefill_rows_per_tile(int kind) { return kind == 0 ? Cfg<0>::R : Cfg<1>::R; }
int prefill_key_tile(int kind) { return kind == 0 ? Cfg<0>::BN : Cfg<1>::BN; }

cudaError_t launch_prefill(const PrefillParams& p, int kind, int grid, cudaStream_t s) {
  if (grid <= 0) return cudaSuccess;
  if (kind == 0) {
    cudaError_t e = cudaFuncSetAttribute(prefill_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Layout<0>::kAlloc);
    if (e != cudaSuccess) return e;
    prefill_kernel<0><<<grid, kThreads, Layout<0>::kAlloc, s>>>(p);
  } else {
    cudaError_t e = cudaFuncSetAttribute(prefill_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Layout<1>::kAlloc);
    if (e != cudaSuccess) return e;
    prefill_kernel<1><<<grid, kThreads, Layout<1>::kAlloc, s>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace mimo
