// Decode: one query token per sequence over the ring (sliding-window layers)
// or paged (global layers) KV cache, split-KV with a combine pass.
//
// Decode streams the cache once: it is HBM-bound (16 FLOP per byte for the
// global layer, 8 for the sliding layer), so the contractions run on
// mma.sync m16n8k16 with the query heads of one KV group as the M rows
// (GQA, "Model techniques map" page, "Grouped-query attention": 16 query heads
// per KV head on global layers, 8 on sliding layers, padded to 16).  Keys are
// streamed with 16-byte cp.async into per-warp double buffers.  The sink logit
// ("Learnable attention sink") joins the final denominator only.
#include <cuda_bf16.h>

#include "common.cuh"
#include "../../include/mimoattn.h"

namespace mimo {

namespace {

constexpr int kWarps = 4;
constexpr int kGroupKeys = 16;
constexpr int kStages = 2;
constexpr int kKStride = kDqk * 2 + 16;  // bytes per key row in smem (padding kills ldmatrix bank conflicts)
constexpr int kVStride = kDv * 2 + 16;
constexpr int kStageBytes = kGroupKeys * (kKStride + kVStride);
constexpr int kQBytes = 16 * kKStride;
constexpr int kSmemBytes = kQBytes + kWarps * kStages * kStageBytes;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
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
__device__ __forceinline__ void mma16816(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// fp16 operands: the rotated dims 0..63 (fp16 in the query tile and in the caches)
__device__ __forceinline__ void mma16816_f16(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ uint32_t smem_u32(const void* p) { return uint32_t(__cvta_generic_to_shared(p)); }

// First visible key and the number of splits of sequence s.
__device__ __forceinline__ void split_range(const DecodeParams& p, int ctx, int* lo, int* nsplit) {
  *lo = p.window > 0 ? max(0, ctx - p.window) : 0;
  *nsplit = (ctx - *lo + p.split_len - 1) / p.split_len;
}

// Cache entry (row index of [entries, Hkv, D]) of position t, or -1 if out of range.
__device__ __forceinline__ long cache_entry(const DecodeParams& p, int s, int t) {
  if (p.cache_kind == MIMO_CACHE_RING) return long(s) * kPage + (t % kPage);
  const int pi = t / kPage;
  const int page = pi < p.max_pages ? p.block_table[long(s) * p.max_pages + pi] : -1;
  if (page < 0 || page >= p.num_pages) return -1;
  return long(page) * kPage + (t % kPage);
}

}  // namespace

__global__ void __launch_bounds__(128, 2) decode_partial_kernel(const DecodeParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int split = blockIdx.x, g = blockIdx.y, s = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ctx = p.seq_lens[s];
  if (ctx < 1 || (p.cache_kind == MIMO_CACHE_RING && p.window > 0 && p.window > kPage)) {
    if (tid == 0 && split == 0) atomicOr(p.status, MIMO_STATUS_BAD_INDEX);
    return;
  }
  int lo, nsplit;
  split_range(p, ctx, &lo, &nsplit);
  if (split >= nsplit) return;
  const int k_begin = lo + split * p.split_len;
  const int k_end = min(k_begin + p.split_len, ctx);
  const int pos = ctx - 1;
  const int G = p.group;

  // ---- rotated query block: 16 rows (the G heads of KV head g, zero padded) x 192
  uint8_t* qs = smem;
  for (int task = tid; task < 16 * 24; task += 128) {
    const int row = task / 24, c = task % 24;
    uint4* dst = reinterpret_cast<uint4*>(qs + row * kKStride);
    if (row >= G) {
      dst[c] = make_uint4(0, 0, 0, 0);
      continue;
    }
    const uint4* src = reinterpret_cast<const uint4*>(p.q + (long(s) * kHq + g * G + row) * kDqk);
    if (c < 4) {
      uint4 a = __ldg(src + c), b = __ldg(src + c + 4);
      rope_chunk_pair(a, b, c, pos, p.rope);
      dst[c] = a;
      dst[c + 4] = b;
    } else if (c >= 8) {
      dst[c] = __ldg(src + c);
    }
  }
  __syncthreads();

  uint32_t qa[12][4];
  {
    const int row = (lane & 7) + ((lane >> 3) & 1) * 8;
    const int col = (lane >> 4) * 8;
#pragma unroll
    for (int kk = 0; kk < 12; ++kk) ldsm_x4(smem_u32(qs + row * kKStride + (16 * kk + col) * 2), qa[kk]);
  }

  uint8_t* stage_base = smem + kQBytes + warp * kStages * kStageBytes;
  const int n_groups = (k_end - k_begin + kGroupKeys - 1) / kGroupKeys;
  // this warp takes groups warp, warp + 4, ...
  auto issue = [&](int gi, int st) {
    uint8_t* kbuf = stage_base + st * kStageBytes;
    uint8_t* vbuf = kbuf + kGroupKeys * kKStride;
    const int t0 = k_begin + gi * kGroupKeys;
    long my_entry = -1;
    if (lane < kGroupKeys && t0 + lane < k_end) my_entry = cache_entry(p, s, t0 + lane);
    if (lane < kGroupKeys && t0 + lane < k_end && my_entry < 0) atomicOr(p.status, MIMO_STATUS_BAD_INDEX);
#pragma unroll 4
    for (int i = 0; i < 20; ++i) {
      const int task = lane + 32 * i;
      const int key = task / 40, c = task % 40;
      const long e = __shfl_sync(0xffffffffu, my_entry, key);
      const bool valid = e >= 0;
      if (c < 24) {
        const uint16_t* src = valid ? p.k_cache + (e * p.hkv + g) * kDqk + c * 8 : p.k_cache;
        cp_async16(smem_u32(kbuf + key * kKStride + c * 16), src, valid);
      } else {
        const int cv = c - 24;
        const uint16_t* src = valid ? p.v_cache + (e * p.hkv + g) * kDv + cv * 8 : p.v_cache;
        cp_async16(smem_u32(vbuf + key * kVStride + cv * 16), src, valid);
      }
    }
  };

  float m_r[2] = {-INFINITY, -INFINITY};
  float l_r[2] = {0.f, 0.f};
  float o[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;

  const int my_groups = n_groups > warp ? (n_groups - warp + kWarps - 1) / kWarps : 0;
  if (my_groups > 0) issue(warp, 0);
  cp_async_commit();
  if (my_groups > 1) issue(warp + kWarps, 1);
  cp_async_commit();

  const float c_log2 = p.scale_log2;
  for (int it = 0; it < my_groups; ++it) {
    const int gi = warp + it * kWarps;
    const int st = it & 1;
    cp_async_wait<1>();
    __syncwarp();
    const uint8_t* kbuf = stage_base + st * kStageBytes;
    const uint8_t* vbuf = kbuf + kGroupKeys * kKStride;
    float acc0[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};
    {
      const int key = (lane & 7) + (lane >> 4) * 8;
      const int dof = ((lane >> 3) & 1) * 8;
#pragma unroll
      for (int kk = 0; kk < 12; ++kk) {
        uint32_t b[4];
        ldsm_x4(smem_u32(kbuf + key * kKStride + (16 * kk + dof) * 2), b);
        if (kk < 4) {  // dims 0..63: rotated, fp16
          mma16816_f16(acc0, qa[kk], b[0], b[1]);
          mma16816_f16(acc1, qa[kk], b[2], b[3]);
        } else {
          mma16816(acc0, qa[kk], b[0], b[1]);
          mma16816(acc1, qa[kk], b[2], b[3]);
        }
      }
    }
    // mask keys past the split end (last group only)
    const int t0 = k_begin + gi * kGroupKeys;
    const int q4 = lane & 3;
    if (t0 + kGroupKeys > k_end) {
      const int c0 = t0 + 2 * q4, c1 = t0 + 8 + 2 * q4;
      if (c0 >= k_end) acc0[0] = acc0[2] = -INFINITY;
      if (c0 + 1 >= k_end) acc0[1] = acc0[3] = -INFINITY;
      if (c1 >= k_end) acc1[0] = acc1[2] = -INFINITY;
      if (c1 + 1 >= k_end) acc1[1] = acc1[3] = -INFINITY;
    }
    float mx0 = fmaxf(fmaxf(acc0[0], acc0[1]), fmaxf(acc1[0], acc1[1]));
    float mx1 = fmaxf(fmaxf(acc0[2], acc0[3]), fmaxf(acc1[2], acc1[3]));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float mn0 = fmaxf(m_r[0], mx0 * c_log2), mn1 = fmaxf(m_r[1], mx1 * c_log2);
    const float a0 = ex2f(m_r[0] - mn0), a1 = ex2f(m_r[1] - mn1);
    m_r[0] = mn0;
    m_r[1] = mn1;
    float p0[4], p1[4];
    p0[0] = ex2f(fmaf(acc0[0], c_log2, -mn0));
    p0[1] = ex2f(fmaf(acc0[1], c_log2, -mn0));
    p0[2] = ex2f(fmaf(acc0[2], c_log2, -mn1));
    p0[3] = ex2f(fmaf(acc0[3], c_log2, -mn1));
    p1[0] = ex2f(fmaf(acc1[0], c_log2, -mn0));
    p1[1] = ex2f(fmaf(acc1[1], c_log2, -mn0));
    p1[2] = ex2f(fmaf(acc1[2], c_log2, -mn1));
    p1[3] = ex2f(fmaf(acc1[3], c_log2, -mn1));
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
      const int key = (lane & 7) + ((lane >> 3) & 1) * 8;
      const int dof = (lane >> 4) * 8;
#pragma unroll
      for (int n2 = 0; n2 < 8; ++n2) {
        uint32_t b[4];
        ldsm_x4_t(smem_u32(vbuf + key * kVStride + (16 * n2 + dof) * 2), b);
        mma16816(o[2 * n2], pa, b[0], b[1]);
        mma16816(o[2 * n2 + 1], pa, b[2], b[3]);
      }
    }
    __syncwarp();
    if (it + 2 < my_groups) issue(gi + 2 * kWarps, st);
    cp_async_commit();
  }
  cp_async_wait<0>();

  // ---- merge the 4 warps (rows = heads)
  l_r[0] += __shfl_xor_sync(0xffffffffu, l_r[0], 1);
  l_r[0] += __shfl_xor_sync(0xffffffffu, l_r[0], 2);
  l_r[1] += __shfl_xor_sync(0xffffffffu, l_r[1], 1);
  l_r[1] += __shfl_xor_sync(0xffffffffu, l_r[1], 2);
  __syncthreads();  // all warps are done with their stage buffers
  float* mw = reinterpret_cast<float*>(smem + kQBytes);  // [4][16]
  float* lw = mw + kWarps * 16;                           // [4][16]
  float* ow = lw + kWarps * 16;                           // [4][16][128]
  const int r0 = lane >> 2, r1 = r0 + 8, q4 = lane & 3;
  if (q4 == 0) {
    mw[warp * 16 + r0] = m_r[0];
    mw[warp * 16 + r1] = m_r[1];
    lw[warp * 16 + r0] = l_r[0];
    lw[warp * 16 + r1] = l_r[1];
  }
#pragma unroll
  for (int nt = 0; nt < 16; ++nt) {
    const int d = nt * 8 + 2 * q4;
    ow[(warp * 16 + r0) * kDv + d] = o[nt][0];
    ow[(warp * 16 + r0) * kDv + d + 1] = o[nt][1];
    ow[(warp * 16 + r1) * kDv + d] = o[nt][2];
    ow[(warp * 16 + r1) * kDv + d + 1] = o[nt][3];
  }
  __syncthreads();
  const int row = tid >> 3, d0 = (tid & 7) * 16;
  if (row >= G) return;
  float M = -INFINITY;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) M = fmaxf(M, mw[w * 16 + row]);
  float wgt[kWarps], L = 0.f;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    wgt[w] = ex2f(mw[w * 16 + row] - M);
    L += wgt[w] * lw[w * 16 + row];
  }
  float acc[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) v += wgt[w] * ow[(w * 16 + row) * kDv + d0 + i];
    acc[i] = v;
  }
  const int h = g * G + row;
  if (nsplit == 1) {
    float M2 = M, L2 = L, f = 1.f;
    if (p.sink) {
      const float sl = p.sink[h] * kLog2e;
      M2 = fmaxf(M, sl);
      f = ex2f(M - M2);
      L2 = L * f + ex2f(sl - M2);
    }
    const float sc = p.v_scale * f / L2;
    uint4 pk[2];
    uint32_t* w32 = reinterpret_cast<uint32_t*>(pk);
#pragma unroll
    for (int i = 0; i < 8; ++i) w32[i] = pack2_bf16(acc[2 * i] * sc, acc[2 * i + 1] * sc);
    uint4* dst = reinterpret_cast<uint4*>(p.out + (long(s) * kHq + h) * kDv + d0);
    dst[0] = pk[0];
    dst[1] = pk[1];
    if (p.lse && d0 == 0) p.lse[long(s) * kHq + h] = (M2 + __log2f(L2)) * kLn2;
  } else {
    float* dst = p.ws_o + ((long(s) * kHq + h) * p.max_splits + split) * kDv + d0;
#pragma unroll
    for (int i = 0; i < 16; i += 4) *reinterpret_cast<float4*>(dst + i) = make_float4(acc[i], acc[i + 1], acc[i + 2], acc[i + 3]);
    if (d0 == 0) {
      float* ml = p.ws_ml + ((long(s) * kHq + h) * p.max_splits + split) * 2;
      ml[0] = M;
      ml[1] = L;
    }
  }
}

// One warp per (sequence, query head): merges the split partials and the sink.
__global__ void __launch_bounds__(256) decode_combine_kernel(const DecodeParams p) {
  const int wid = int((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (wid >= p.batch * kHq) return;
  const int s = wid / kHq, h = wid % kHq;
  const int ctx = p.seq_lens[s];
  if (ctx < 1) return;
  int lo, nsplit;
  split_range(p, ctx, &lo, &nsplit);
  if (nsplit <= 1) return;  // written by the partial kernel
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
    const float w = ex2f(ml[2 * i] - M);
    L += w * ml[2 * i + 1];
    const float4 v = *reinterpret_cast<const float4*>(ob + long(i) * kDv + lane * 4);
    acc.x += w * v.x;
    acc.y += w * v.y;
    acc.z += w * v.z;
    acc.w += w * v.w;
  }
  if (p.sink) L += ex2f(sl - M);
  const float sc = p.v_scale / L;
  uint2 pk;
  pk.x = pack2_bf16(acc.x * sc, acc.y * sc);
  pk.y = pack2_bf16(acc.z * sc, acc.w * sc);
  *reinterpret_cast<uint2*>(p.out + (long(s) * kHq + h) * kDv + lane * 4) = pk;
  if (p.lse && lane == 0) p.lse[long(s) * kHq + h] = (M + __log2f(L)) * kLn2;
}

cudaError_t launch_decode(const DecodeParams& p, cudaStream_t s) {
  cudaError_t e0 = cudaFuncSetAttribute(decode_partial_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e0 != cudaSuccess) return e0;
  dim3 grid(p.max_splits, p.hkv, p.batch);
  decode_partial_kernel<<<grid, 128, kSmemBytes, s>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || p.max_splits <= 1) return e;
  const long warps = long(p.batch) * kHq;
  decode_combine_kernel<<<unsigned((warps * 32 + 255) / 256), 256, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace mimo
