// KV append: rotate the first 64 dims of each new key at its position and
// store key and value into the ring or paged cache.  Cache rows hold the key
// as dims 0..63 rotated in IEEE fp16 and dims 64..191 in bf16 (the input
// format), and the value in bf16; or, for an E4M3 cache, every element as one
// E4M3 byte scaled by 1 / (its KV head's dequantisation scale).
//
// Cache layout follows the serving pages: window-sized KV for the sliding
// layers (gaudi-cookbook "MiMo-V2.6-Flash-RL", "Launch": window-sized KV for
// the 39 sliding layers) kept here as a 128-slot ring per sequence, and paged
// KV with block size 128 for the global layers (same page, "--block-size 128").
#include "common.cuh"
#include "../../include/mimoattn.h"

namespace mimo {

// One warp per (token, kv head).  Lanes 0..3 rotate the chunk pairs (u, u+4) of
// dims 0..63; lanes 8..23 copy chunks 8..23 (dims 64..191); lanes 0..15 copy V.
__global__ void __launch_bounds__(256) kv_append_kernel(const AppendParams p) {
  const int warp = int((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (warp >= p.num_tokens * p.hkv) return;
  const int t = warp / p.hkv, g = warp % p.hkv;
  const int pos = p.pos[t], s = p.seq_idx[t];
  long entry;
  if (s < 0 || s >= p.num_seqs || pos < 0) {
    if (lane == 0) atomicOr(p.status, MIMO_STATUS_BAD_INDEX);
    return;
  }
  if (p.cache_kind == MIMO_CACHE_RING) {
    entry = long(s) * p.ring_slots + (pos % p.ring_slots);
  } else {
    const int pi = pos / kPage;
    const int page = pi < p.max_pages ? p.block_table[long(s) * p.max_pages + pi] : -1;
    if (page < 0 || page >= p.num_pages) {
      if (lane == 0) atomicOr(p.status, MIMO_STATUS_BAD_INDEX);
      return;
    }
    entry = long(page) * kPage + (pos % kPage);
  }
  const uint4* ks = reinterpret_cast<const uint4*>(p.k_new + (long(t) * p.hkv + g) * kDqk);
  if (p.fp8) {
    // E4M3 rows: each element divided by its KV head's dequantisation scale, rounded to
    // nearest even and saturated (the rotation itself in fp32).  A scale that is not finite
    // and positive would store inf / NaN or sign-flipped codes: skip the row and report it.
    const float kdq = p.k_dequant[g], vdq = p.v_dequant[g];
    if (!(kdq > 0.f && kdq < INFINITY && vdq > 0.f && vdq < INFINITY)) {
      if (lane == 0) atomicOr(p.status, MIMO_STATUS_BAD_SCALE);
      return;
    }
    const float kq = 1.f / kdq, vq = 1.f / vdq;
    uint8_t* k8 = reinterpret_cast<uint8_t*>(p.k_cache) + (entry * p.hkv + g) * kDqk;
    uint8_t* v8 = reinterpret_cast<uint8_t*>(p.v_cache) + (entry * p.hkv + g) * kDv;
    auto pack8 = [](const float* x, float sc) {
      return make_uint2(uint32_t(e4m3x2_from_f32(x[0] * sc, x[1] * sc)) | (uint32_t(e4m3x2_from_f32(x[2] * sc, x[3] * sc)) << 16),
                        uint32_t(e4m3x2_from_f32(x[4] * sc, x[5] * sc)) | (uint32_t(e4m3x2_from_f32(x[6] * sc, x[7] * sc)) << 16));
    };
    auto widen8 = [](const uint4& c, float* x) {
      const uint32_t w[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        x[2 * i] = lo_bf16(w[i]);
        x[2 * i + 1] = hi_bf16(w[i]);
      }
    };
    if (lane < 4) {
      // dims 8u..8u+7 pair with 8u+32..8u+39 (frequency index 8u + i)
      float x[8], y[8], xr[8], yr[8];
      widen8(__ldg(ks + lane), x);
      widen8(__ldg(ks + lane + 4), y);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float c, sn;
        rope_cos_sin(pos, p.rope.inv_freq[8 * lane + i], &c, &sn);
        xr[i] = x[i] * c - y[i] * sn;
        yr[i] = y[i] * c + x[i] * sn;
      }
      *reinterpret_cast<uint2*>(k8 + 8 * lane) = pack8(xr, kq);
      *reinterpret_cast<uint2*>(k8 + 32 + 8 * lane) = pack8(yr, kq);
    } else if (lane >= 8 && lane < 24) {
      float x[8];
      widen8(__ldg(ks + lane), x);
      *reinterpret_cast<uint2*>(k8 + 8 * lane) = pack8(x, kq);
    }
    if (lane < 16) {
      float x[8];
      widen8(__ldg(reinterpret_cast<const uint4*>(p.v_new + (long(t) * p.hkv + g) * kDv) + lane), x);
      *reinterpret_cast<uint2*>(v8 + 8 * lane) = pack8(x, vq);
    }
    return;
  }
  uint4* kd = reinterpret_cast<uint4*>(p.k_cache + (entry * p.hkv + g) * kDqk);
  if (lane < 4) {
    uint4 lo = __ldg(ks + lane), hi = __ldg(ks + lane + 4);
    float amax = 0.f;
    rope_chunk_pair(lo, hi, lane, pos, p.rope, amax);
    if (amax > kF16Max) atomicOr(p.status, MIMO_STATUS_RANGE);
    kd[lane] = lo;
    kd[lane + 4] = hi;
  } else if (lane >= 8 && lane < 24) {
    kd[lane] = __ldg(ks + lane);
  }
  if (lane < 16) {
    const uint4* vs = reinterpret_cast<const uint4*>(p.v_new + (long(t) * p.hkv + g) * kDv);
    uint4* vd = reinterpret_cast<uint4*>(p.v_cache + (entry * p.hkv + g) * kDv);
    vd[lane] = __ldg(vs + lane);
  }
}

cudaError_t launch_kv_append(const AppendParams& p, cudaStream_t s) {
  const long warps = long(p.num_tokens) * p.hkv;
  if (warps == 0) return cudaSuccess;
  const int block = 256;
  const long grid = (warps * 32 + block - 1) / block;
  kv_append_kernel<<<unsigned(grid), block, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace mimo
