// Decode: one query token per sequence over the ring (sliding-window layers)
// or paged (global layers) KV cache, split-KV with a combine pass.
//
// Decode streams the cache once: it is HBM-bound (16 FLOP per byte for the
// global layer, 8 for the sliding layer), so the contractions run on
// mma.sync m16n8k16 with the query heads of one KV group as the M rows
// (GQA, "Model techniques map" page, "Grouped-query attention": 16 query heads
// per KV head on global layers, 8 on sliding layers, padded to 16).  The sink
// logit ("Learnable attention sink") joins the final denominator only.
//
// Persistent kernel: one CTA per SM walks work units (split, sequence, KV head).
// Warp 0 streams 64-key K/V tiles with TMA (128-byte swizzle, 4 stages of 40 KB,
// page ids fetched once per unit); warps 1..4 each take 16 keys of every tile.
// Each compute warp builds its query fragments straight from global memory and
// applies the partial RoPE in registers (dims j and j+32 land in the same
// thread).  A ring cache is read in slot order with each slot's position
// recovered from the context length: attention does not depend on key order.
#include <cuda_bf16.h>

#include "common.cuh"
#include "ptx.cuh"
#include "../../include/mimoattn.h"

namespace mimo {

namespace {

constexpr int kTile = 64;  // keys per TMA tile
constexpr int kStages = 4;
constexpr int kThreads = 160;
constexpr int kKChunk = kTile * 128;                    // 64 keys x 64 dims, 2-byte elements
constexpr int kStageBytes = 3 * kKChunk + 2 * kKChunk;  // K (3 chunks) + V (2 chunks)
constexpr int kOffMerge = kStages * kStageBytes;
constexpr int kMergeBytes = 4 * 16 * 4 * 2 + 4 * 16 * kDv * 4;
constexpr int kOffBar = kOffMerge + kMergeBytes;
constexpr int kSmemBytes = kOffBar + 16 * 8 + 1024;
static_assert(kSmemBytes <= 232448, "shared memory budget");
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

struct Unit {
  int s, g, split;
  int ctx, k_begin, k_end;  // keys [k_begin, k_end) of this split
  int t0, nt;               // tiles (absolute 64-key tiles, or the two ring halves)
};

// Work unit u of the dense space [split][sequence][kv head]; false if it has no keys.
__device__ __forceinline__ bool unit_at(const DecodeParams& p, int u, Unit& U) {
  const int per_split = p.batch * p.hkv;
  U.split = u / per_split;
  const int rem = u - U.split * per_split;
  U.s = rem / p.hkv;
  U.g = rem - U.s * p.hkv;
  U.ctx = p.seq_lens[U.s];
  if (U.ctx < 1) return false;
  const int lo = p.window > 0 ? max(0, U.ctx - p.window) : 0;
  U.k_begin = lo + U.split * p.split_len;
  if (U.k_begin >= U.ctx) return false;
  U.k_end = min(U.k_begin + p.split_len, U.ctx);
  if (p.cache_kind == MIMO_CACHE_RING) {
    U.t0 = 0;
    U.nt = 2;  // the 128 slots, in slot order
  } else {
    U.t0 = U.k_begin / kTile;
    U.nt = (U.k_end - 1) / kTile - U.t0 + 1;
  }
  return true;
}

}  // namespace

__global__ void __launch_bounds__(kThreads, 1) decode_kernel(const __grid_constant__ DecodeParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t bar0 = sbase + kOffBar;
  auto full = [&](int i) { return bar0 + 8 * i; };
  auto empty = [&](int i) { return bar0 + 8 * (kStages + i); };
  const uint32_t merge_ready = bar0 + 8 * (2 * kStages);
  const uint32_t merge_free = bar0 + 8 * (2 * kStages + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffBar + 8 * (2 * kStages + 2));
  unsigned* status = p.status;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(full(i), 1);
      mbar_init(empty(i), 4);
    }
    mbar_init(merge_ready, 128);
    mbar_init(merge_free, 128);
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const int n_units = p.batch * p.hkv * p.max_splits;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch(&p.tm_k);
      tma_prefetch(&p.tm_v);
    }
    int it = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
      Unit U;
      if (!unit_at(p, u, U)) continue;
      // cache row of each tile of the unit (lane i: tile i); a unit spans at most 32 tiles
      int row_l = 0;
      if (lane < U.nt) {
        if (p.cache_kind == MIMO_CACHE_RING) {
          row_l = U.s * kPage + kTile * lane;
        } else {
          const int pi = (U.t0 + lane) * kTile / kPage;
          int page = pi < p.max_pages ? p.block_table[long(U.s) * p.max_pages + pi] : -1;
          if (page < 0 || page >= p.num_pages) {
            atomicOr(status, MIMO_STATUS_BAD_INDEX);
            page = 0;
          }
          row_l = page * kPage + ((U.t0 + lane) * kTile) % kPage;
        }
      }
      for (int t = 0; t < U.nt; ++t, ++it) {
        const int row = __shfl_sync(0xffffffffu, row_l, t);
        const int st = it % kStages;
        if (it >= kStages &&
            !(ok = __all_sync(0xffffffffu, mbar_wait(empty(st), ((it / kStages) - 1) & 1, abort_flag, status,
                                                     MIMO_STATUS_TIMEOUT))))
          break;
        if (lane == 0) {
          const uint32_t dst = sbase + st * kStageBytes;
          mbar_expect_tx(full(st), kStageBytes);
          tma_load_3d(dst, &p.tm_k, full(st), 0, U.g, row);
          tma_load_3d(dst + kKChunk, &p.tm_k, full(st), 64, U.g, row);
          tma_load_3d(dst + 2 * kKChunk, &p.tm_k, full(st), 128, U.g, row);
          tma_load_3d(dst + 3 * kKChunk, &p.tm_v, full(st), 0, U.g, row);
          tma_load_3d(dst + 4 * kKChunk, &p.tm_v, full(st), 64, U.g, row);
        }
        __syncwarp();
      }
    }
    if (!ok && lane == 0) {
      // let copies already in flight land before the CTA leaves
      int dummy = 0;
      for (int i = 0; i < kStages; ++i) mbar_wait(full(i), 0, &dummy, nullptr, 0, 50000000ull);
    }
    return;
  }

  // ------------------------------------------------------------ compute warps 1..4
  const int cw = warp - 1;
  const int tid = threadIdx.x - 32;  // 0..127
  const int G = p.group;
  const int q4 = lane & 3, r0 = lane >> 2, r1 = r0 + 8;
  const float c_log2 = p.scale_log2;
  float* mw = reinterpret_cast<float*>(smem + kOffMerge);  // [4][16]
  float* lw = mw + 4 * 16;                                 // [4][16]
  float* ow = lw + 4 * 16;                                 // [4][16][128]
  auto wait_w = [&](uint32_t bar, uint32_t parity) -> bool {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, status, MIMO_STATUS_TIMEOUT));
  };
  int it = 0, n_done = 0;
  bool ok = true;
  for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
    Unit U;
    if (!unit_at(p, u, U)) continue;
    const int pos = U.ctx - 1;
    // ---- query fragments (A of m16n8k16) for the G heads of KV head g, RoPE in registers
    uint32_t qa[12][4];
    {
      const uint16_t* q0 = p.q + (long(U.s) * kHq + U.g * G) * kDqk;
      const bool v0 = r0 < G, v1 = r1 < G;
#pragma unroll
      for (int kk = 0; kk < 12; ++kk) {
        const int c = 16 * kk + 2 * q4;
        qa[kk][0] = v0 ? *reinterpret_cast<const uint32_t*>(q0 + r0 * kDqk + c) : 0u;
        qa[kk][1] = v1 ? *reinterpret_cast<const uint32_t*>(q0 + r1 * kDqk + c) : 0u;
        qa[kk][2] = v0 ? *reinterpret_cast<const uint32_t*>(q0 + r0 * kDqk + c + 8) : 0u;
        qa[kk][3] = v1 ? *reinterpret_cast<const uint32_t*>(q0 + r1 * kDqk + c + 8) : 0u;
      }
      // dims j < 32 (k-steps 0, 1) pair with dims j + 32 (k-steps 2, 3) in the same register slot
#pragma unroll
      for (int kk = 0; kk < 2; ++kk)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j0 = 16 * kk + 2 * q4 + ((e & 2) ? 8 : 0);
          float c0, s0, c1, s1;
          rope_cos_sin(pos, p.rope.inv_freq[j0], &c0, &s0);
          rope_cos_sin(pos, p.rope.inv_freq[j0 + 1], &c1, &s1);
          const uint32_t xw = qa[kk][e], yw = qa[kk + 2][e];
          const float x0 = lo_bf16(xw), x1 = hi_bf16(xw), y0 = lo_bf16(yw), y1 = hi_bf16(yw);
          qa[kk][e] = pack2_f16(x0 * c0 - y0 * s0, x1 * c1 - y1 * s1);
          qa[kk + 2][e] = pack2_f16(y0 * c0 + x0 * s0, y1 * c1 + x1 * s1);
        }
    }
    float m_r[2] = {-INFINITY, -INFINITY};
    float l_r[2] = {0.f, 0.f};
    float o[16][4];
#pragma unroll
    for (int i = 0; i < 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;

    for (int t = 0; t < U.nt; ++t, ++it) {
      const int st = it % kStages;
      if (!(ok = wait_w(full(st), (it / kStages) & 1))) break;
      const uint32_t kb = sbase + st * kStageBytes;
      const uint32_t vb = kb + 3 * kKChunk;
      float acc0[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};
      {
        // B fragments of K^T: matrices (keys 0-7 | 8-15) x (dims lo 8 | hi 8) of this warp's 16 keys;
        // rows are 128-byte swizzled (16-byte unit u of row k sits at u ^ (k & 7))
        const int key = 16 * cw + (lane & 7) + (lane >> 4) * 8;
        const int dhalf = (lane >> 3) & 1;
#pragma unroll
        for (int kk = 0; kk < 12; ++kk) {
          const int unit16 = ((kk & 3) * 2 + dhalf) ^ (key & 7);
          uint32_t b[4];
          ldsm_x4(kb + (kk >> 2) * kKChunk + key * 128 + unit16 * 16, b);
          if (kk < 4) {
            mma_f16(acc0, qa[kk], b[0], b[1]);
            mma_f16(acc1, qa[kk], b[2], b[3]);
          } else {
            mma_bf16(acc0, qa[kk], b[0], b[1]);
            mma_bf16(acc1, qa[kk], b[2], b[3]);
          }
        }
      }
      // positions of this thread's four key columns and their visibility
      bool vis[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int col = 16 * cw + ((e & 2) ? 8 : 0) + 2 * q4 + (e & 1);  // within the 64-key tile
        int kp;
        if (p.cache_kind == MIMO_CACHE_RING) {
          const int slot = kTile * t + col;
          const int base = U.ctx - kPage;  // the ring holds positions base .. ctx-1
          kp = base + (((slot - base) % kPage) + kPage) % kPage;
        } else {
          kp = (U.t0 + t) * kTile + col;
        }
        vis[e] = kp >= U.k_begin && kp < U.k_end;
      }
      if (!vis[0]) acc0[0] = acc0[2] = -INFINITY;
      if (!vis[1]) acc0[1] = acc0[3] = -INFINITY;
      if (!vis[2]) acc1[0] = acc1[2] = -INFINITY;
      if (!vis[3]) acc1[1] = acc1[3] = -INFINITY;
      float mx0 = fmaxf(fmaxf(acc0[0], acc0[1]), fmaxf(acc1[0], acc1[1]));
      float mx1 = fmaxf(fmaxf(acc0[2], acc0[3]), fmaxf(acc1[2], acc1[3]));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
      const float mn0 = fmaxf(m_r[0], mx0 * c_log2), mn1 = fmaxf(m_r[1], mx1 * c_log2);
      // all keys of this warp's share of a tile may be masked (tile edges): reference 0 then
      const float mu0 = mn0 == -INFINITY ? 0.f : mn0, mu1 = mn1 == -INFINITY ? 0.f : mn1;
      const float a0 = ex2(m_r[0] - mu0), a1 = ex2(m_r[1] - mu1);
      m_r[0] = mn0;
      m_r[1] = mn1;
      float p0[4], p1[4];
      p0[0] = ex2(fmaf(acc0[0], c_log2, -mu0));
      p0[1] = ex2(fmaf(acc0[1], c_log2, -mu0));
      p0[2] = ex2(fmaf(acc0[2], c_log2, -mu1));
      p0[3] = ex2(fmaf(acc0[3], c_log2, -mu1));
      p1[0] = ex2(fmaf(acc1[0], c_log2, -mu0));
      p1[1] = ex2(fmaf(acc1[1], c_log2, -mu0));
      p1[2] = ex2(fmaf(acc1[2], c_log2, -mu1));
      p1[3] = ex2(fmaf(acc1[3], c_log2, -mu1));
      l_r[0] = l_r[0] * a0 + p0[0] + p0[1] + p1[0] + p1[1];
      l_r[1] = l_r[1] * a1 + p0[2] + p0[3] + p1[2] + p1[3];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        o[i][0] *= a0;
        o[i][1] *= a0;
        o[i][2] *= a1;
        o[i][3] *= a1;
      }
      uint32_t pa[4];
      pa[0] = pack2_bf16(p0[0], p0[1]);
      pa[1] = pack2_bf16(p0[2], p0[3]);
      pa[2] = pack2_bf16(p1[0], p1[1]);
      pa[3] = pack2_bf16(p1[2], p1[3]);
      {
        // B fragments of V (trans): matrices (keys 0-7 | 8-15) x (dims d0 .. d0+7 | d0+8 ..)
        const int key = 16 * cw + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int dq = lane >> 4;
#pragma unroll
        for (int n2 = 0; n2 < 8; ++n2) {
          const int unit16 = ((n2 & 3) * 2 + dq) ^ (key & 7);
          uint32_t b[4];
          ldsm_x4_t(vb + (n2 >> 2) * kKChunk + key * 128 + unit16 * 16, b);
          mma_bf16(o[2 * n2], pa, b[0], b[1]);
          mma_bf16(o[2 * n2 + 1], pa, b[2], b[3]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty(st));
    }
    if (!ok) break;

    // ---- merge the 4 warps (rows = heads) and write the unit's result
    l_r[0] += __shfl_xor_sync(0xffffffffu, l_r[0], 1);
    l_r[0] += __shfl_xor_sync(0xffffffffu, l_r[0], 2);
    l_r[1] += __shfl_xor_sync(0xffffffffu, l_r[1], 1);
    l_r[1] += __shfl_xor_sync(0xffffffffu, l_r[1], 2);
    if (n_done > 0 && !(ok = wait_w(merge_free, (n_done - 1) & 1))) break;
    if (q4 == 0) {
      mw[cw * 16 + r0] = m_r[0];
      mw[cw * 16 + r1] = m_r[1];
      lw[cw * 16 + r0] = l_r[0];
      lw[cw * 16 + r1] = l_r[1];
    }
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
      const int d = nt * 8 + 2 * q4;
      *reinterpret_cast<float2*>(ow + (cw * 16 + r0) * kDv + d) = make_float2(o[nt][0], o[nt][1]);
      *reinterpret_cast<float2*>(ow + (cw * 16 + r1) * kDv + d) = make_float2(o[nt][2], o[nt][3]);
    }
    mbar_arrive(merge_ready);
    if (!(ok = wait_w(merge_ready, n_done & 1))) break;
    {
      const int row = tid >> 3, d0 = (tid & 7) * 16;
      if (row < G) {
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < 4; ++w) M = fmaxf(M, mw[w * 16 + row]);
        const float Mu = M == -INFINITY ? 0.f : M;
        float wgt[4], L = 0.f;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          wgt[w] = ex2(mw[w * 16 + row] - Mu);
          L += wgt[w] * lw[w * 16 + row];
        }
        float acc[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          float v = 0.f;
#pragma unroll
          for (int w = 0; w < 4; ++w) v += wgt[w] * ow[(w * 16 + row) * kDv + d0 + i];
          acc[i] = v;
        }
        const int h = U.g * G + row;
        if (p.max_splits == 1) {
          float M2 = Mu, L2 = L, f = 1.f;
          if (p.sink) {
            const float sl = p.sink[h] * kLog2e;
            M2 = fmaxf(Mu, sl);
            f = ex2(Mu - M2);
            L2 = L * f + ex2(sl - M2);
          }
          const float sc = p.v_scale * f / L2;
          uint4* dst = reinterpret_cast<uint4*>(p.out + (long(U.s) * kHq + h) * kDv + d0);
#pragma unroll
          for (int i = 0; i < 2; ++i)
            dst[i] = make_uint4(pack2_bf16(acc[8 * i] * sc, acc[8 * i + 1] * sc),
                                pack2_bf16(acc[8 * i + 2] * sc, acc[8 * i + 3] * sc),
                                pack2_bf16(acc[8 * i + 4] * sc, acc[8 * i + 5] * sc),
                                pack2_bf16(acc[8 * i + 6] * sc, acc[8 * i + 7] * sc));
          if (p.lse && d0 == 0) p.lse[long(U.s) * kHq + h] = (M2 + __log2f(L2)) * kLn2;
        } else {
          float* dst = p.ws_o + ((long(U.s) * kHq + h) * p.max_splits + U.split) * kDv + d0;
#pragma unroll
          for (int i = 0; i < 16; i += 4)
            *reinterpret_cast<float4*>(dst + i) = make_float4(acc[i], acc[i + 1], acc[i + 2], acc[i + 3]);
          if (d0 == 0) {
            float* ml = p.ws_ml + ((long(U.s) * kHq + h) * p.max_splits + U.split) * 2;
            ml[0] = M;
            ml[1] = L;
          }
        }
      }
    }
    mbar_arrive(merge_free);
    ++n_done;
  }
}

// One warp per (sequence, query head): merges the split partials and the sink.
__global__ void __launch_bounds__(256) decode_combine_kernel(const __grid_constant__ DecodeParams p) {
  const int wid = int((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (wid >= p.batch * kHq) return;
  const int s = wid / kHq, h = wid % kHq;
  const int ctx = p.seq_lens[s];
  if (ctx < 1) {
    if (lane == 0 && h == 0) atomicOr(p.status, MIMO_STATUS_BAD_INDEX);
    return;
  }
  const int lo = p.window > 0 ? max(0, ctx - p.window) : 0;
  const int nsplit = (ctx - lo + p.split_len - 1) / p.split_len;
  const float* ml = p.ws_ml + (long(s) * kHq + h) * p.max_splits * 2;
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
  const float* ob = p.ws_o + (long(s) * kHq + h) * p.max_splits * kDv;
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
  *reinterpret_cast<uint2*>(p.out + (long(s) * kHq + h) * kDv + lane * 4) = pk;
  if (p.lse && lane == 0) p.lse[long(s) * kHq + h] = (M + __log2f(L)) * kLn2;
}

cudaError_t launch_decode(const DecodeParams& p, int sms, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  const long units = long(p.batch) * p.hkv * p.max_splits;
  const int grid = int(units < sms ? units : sms);
  decode_kernel<<<grid, kThreads, kSmemBytes, s>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess || p.max_splits <= 1) return e;
  const long warps = long(p.batch) * kHq;
  decode_combine_kernel<<<unsigned((warps * 32 + 255) / 256), 256, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace mimo
