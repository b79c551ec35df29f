// Float64 CPU oracle of the MiMo-V2.6-Flash hybrid attention forward.
//
// TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the bench's
// CPU-baseline / reference legs may load this library.  It shares no code,
// header, table or helper with the CUDA path under global_attention_attn_b200/.
//
// What it computes is the attention layer as the model pages state it:
//  * radixark miles docs "MiMo-V2.6-Flash", section 1 "Key highlights": 39
//    sliding-window layers (window 128, learnable attention sink) and 9 global
//    layers; 8 vs 4 KV heads; RoPE bases 1e4 vs 1e7; 192-dim Q/K, 128-dim V,
//    V scaled by 0.707; partial RoPE on 64 of 192 dims.
//  * same page, section 5.4 "Notable quirks": the window convention.  This
//    oracle takes `window` = number of keys in total including the query
//    itself (128 for the HF modeling code), so the SGLang convention is window 129.
//  * "Model techniques map" page, "Grouped-query attention": repeat_kv, so
//    query head h reads KV head h / (Hq / Hkv).
//  * same page, "Learnable attention sink": a per-query-head logit appended as
//    an extra column before the softmax; its column carries no value.
//  * same page, "Partial RoPE": the rotary part is the first rope_dim dims of
//    each head, the rest passes through.  Pairing (NeoX rotate-half) and
//    frequencies base^(-2j/rope_dim) are the "default" rope type.
//  * gaudi-cookbook "MiMo-V2.6-Flash-RL", "Required fixes": rotary angles are
//    taken in float64 because the fastest angle equals the position.
//
// Inputs are bf16 bit patterns widened exactly to double; every step runs in
// double.  For query row at position p and head h:
//   keys K = { t : t <= p and (window == 0 or p - t < window) }
//   z_t = scale * rope(q, p) . k_t      (k_t rotated at t unless it comes from a cache,
//                                        where it is stored rotated already)
//   M = max(z_t, sink_h);  Z = sum exp(z_t - M) + exp(sink_h - M)
//   out = v_scale * sum exp(z_t - M) v_t / Z;   lse = M + ln Z
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

namespace {

inline double bf16_to_double(uint16_t b) {
  uint32_t u = uint32_t(b) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return double(f);
}

// IEEE 754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits.
inline double f16_to_double(uint16_t h) {
  const int sign = (h >> 15) & 1, e = (h >> 10) & 0x1F, f = h & 0x3FF;
  double v;
  if (e == 0) v = std::ldexp(double(f), -24);                       // zero / subnormal
  else if (e == 31) v = f ? NAN : INFINITY;
  else v = std::ldexp(double(f | 0x400), e - 25);                   // (1 + f/1024) * 2^(e-15)
  return sign ? -v : v;
}

// OCP 8-bit floating point, E4M3 ("FP8 E4M3"): 1 sign bit, 4 exponent bits
// (bias 7), 3 mantissa bits; exponent 0 holds zero and the subnormals m/8 * 2^-6;
// no infinities; exponent 15 with mantissa 7 is NaN, so the largest value is
// 1.75 * 2^8 = 448.
inline double e4m3_to_double(uint8_t c) {
  const int sign = c >> 7, e = (c >> 3) & 0xF, m = c & 7;
  double v;
  if (e == 0) v = std::ldexp(double(m), -9);                        // (m / 8) * 2^-6
  else if (e == 15 && m == 7) v = NAN;
  else v = std::ldexp(double(8 + m), e - 10);                        // (1 + m/8) * 2^(e-7)
  return sign ? -v : v;
}

}  // namespace

extern "C" {

double oracle_e4m3_to_double(int code) { return e4m3_to_double(uint8_t(code)); }

// Layer description plus where each sequence's keys live.  Keys at positions
// [new_pos0[s], new_pos0[s] + new_len[s]) come from the contiguous pre-RoPE
// arrays k_new / v_new (row new_row0[s] + (pos - new_pos0[s])); keys at positions
// below new_pos0[s] come from the cache (stored rotated):
//   cache_kind 1 (paged): page block_table[s * max_pages + pos / page_size], slot pos % page_size
//   cache_kind 2 (ring):  entry s * page_size + pos % page_size
// Cache rows use the library's cache format: key dims < rope_dim are IEEE
// fp16 bit patterns (the rotated part), the other key dims and the values bf16
// (cache_dtype 0); or every key and value element is an E4M3 byte that
// dequantises to code * k_dequant[g] (keys) / code * v_dequant[g] (values) (cache_dtype 1).
typedef struct {
  int hq, hkv, dqk, dv, rope_dim;
  double rope_base, softmax_scale, v_scale;
  int window;
  const float* sink;
  int num_seqs;
  const int32_t* q_row0;
  const int32_t* q_len;
  const int32_t* q_pos0;
  const uint16_t* k_new;
  const uint16_t* v_new;
  const int32_t* new_row0;
  const int32_t* new_pos0;
  const int32_t* new_len;
  int cache_kind;
  const uint16_t* k_cache;
  const uint16_t* v_cache;
  int page_size;
  const int32_t* block_table;
  int max_pages;
  int cache_dtype;
  const float* k_dequant;  // [hkv], cache_dtype 1
  const float* v_dequant;
} oracle_layer;

// Partial NeoX rotation of one head vector x[0..d) at position pos, in double.
// Pairs (j, j + rope_dim/2) for j < rope_dim/2, angle pos * base^(-2j/rope_dim).
void oracle_rope(const double* x, int d, int rope_dim, double base, double pos, double* out) {
  const int half = rope_dim / 2;
  for (int i = 0; i < d; ++i) out[i] = x[i];
  for (int j = 0; j < half; ++j) {
    const double theta = pos * std::pow(base, -2.0 * double(j) / double(rope_dim));
    const double c = std::cos(theta), s = std::sin(theta);
    out[j] = x[j] * c - x[j + half] * s;
    out[j + half] = x[j + half] * c + x[j] * s;
  }
}

}  // extern "C"

namespace {

struct Ctx {
  const oracle_layer* L;
  const uint16_t* q;
  // per sequence: rotated copies (double) of the contiguous new keys
  std::vector<std::vector<double>> krot;  // [s][(pos - new_pos0) * hkv * dqk + ...]
};

// Key position p of sequence s, KV head g: fills k (double, rotated) and/or v
// (double) when the pointers are non-null.  Returns false if the position is
// not held anywhere.
bool fetch_key(const Ctx& C, int s, int p, int g, double* k, double* v) {
  const oracle_layer* L = C.L;
  const int np0 = L->new_pos0 ? L->new_pos0[s] : 0;
  const int nlen = L->new_len ? L->new_len[s] : 0;
  if (p >= np0 && p < np0 + nlen) {
    if (k) std::memcpy(k, &C.krot[s][(size_t(p - np0) * L->hkv + g) * L->dqk], sizeof(double) * L->dqk);
    if (v) {
      const size_t row = size_t(L->new_row0[s]) + size_t(p - np0);
      const uint16_t* vp = L->v_new + (row * L->hkv + g) * L->dv;
      for (int i = 0; i < L->dv; ++i) v[i] = bf16_to_double(vp[i]);
    }
    return true;
  }
  if (p < np0 && L->cache_kind != 0) {
    size_t entry;
    if (L->cache_kind == 1) {
      const int page = L->block_table[size_t(s) * L->max_pages + p / L->page_size];
      entry = size_t(page) * L->page_size + (p % L->page_size);
    } else {
      entry = size_t(s) * L->page_size + (p % L->page_size);
    }
    if (L->cache_dtype == 1) {
      const uint8_t* kp = reinterpret_cast<const uint8_t*>(L->k_cache) + (entry * L->hkv + g) * L->dqk;
      const uint8_t* vp = reinterpret_cast<const uint8_t*>(L->v_cache) + (entry * L->hkv + g) * L->dv;
      if (k)
        for (int i = 0; i < L->dqk; ++i) k[i] = e4m3_to_double(kp[i]) * double(L->k_dequant[g]);
      if (v)
        for (int i = 0; i < L->dv; ++i) v[i] = e4m3_to_double(vp[i]) * double(L->v_dequant[g]);
      return true;
    }
    const uint16_t* kp = L->k_cache + (entry * L->hkv + g) * L->dqk;
    const uint16_t* vp = L->v_cache + (entry * L->hkv + g) * L->dv;
    if (k)
      for (int i = 0; i < L->dqk; ++i) k[i] = i < L->rope_dim ? f16_to_double(kp[i]) : bf16_to_double(kp[i]);
    if (v)
      for (int i = 0; i < L->dv; ++i) v[i] = bf16_to_double(vp[i]);
    return true;
  }
  return false;
}

int prepare(Ctx& C) {
  const oracle_layer* L = C.L;
  C.krot.assign(L->num_seqs, {});
  std::vector<double> x(L->dqk), y(L->dqk);
  for (int s = 0; s < L->num_seqs; ++s) {
    const int nlen = L->new_len ? L->new_len[s] : 0;
    if (nlen <= 0) continue;
    C.krot[s].resize(size_t(nlen) * L->hkv * L->dqk);
    for (int t = 0; t < nlen; ++t) {
      const size_t row = size_t(L->new_row0[s]) + t;
      for (int g = 0; g < L->hkv; ++g) {
        const uint16_t* kp = L->k_new + (row * L->hkv + g) * L->dqk;
        for (int i = 0; i < L->dqk; ++i) x[i] = bf16_to_double(kp[i]);
        oracle_rope(x.data(), L->dqk, L->rope_dim, L->rope_base, double(L->new_pos0[s] + t), y.data());
        std::memcpy(&C.krot[s][(size_t(t) * L->hkv + g) * L->dqk], y.data(), sizeof(double) * L->dqk);
      }
    }
  }
  return 0;
}

// One (query row, head): the definition, two passes (max, then sums).
// If online != 0 the same quantity is accumulated in one pass with a running
// maximum (the streaming form); it must agree with the two-pass form.
int one_row(const Ctx& C, int s, int i, int h, int online, double* out, double* lse) {
  const oracle_layer* L = C.L;
  const int G = L->hq / L->hkv;
  const int g = h / G;
  const int p = L->q_pos0[s] + i;
  const size_t qrow = size_t(L->q_row0[s]) + i;
  std::vector<double> qx(L->dqk), qr(L->dqk), k(L->dqk), v(L->dv);
  const uint16_t* qp = C.q + (qrow * L->hq + h) * L->dqk;
  for (int d = 0; d < L->dqk; ++d) qx[d] = bf16_to_double(qp[d]);
  oracle_rope(qx.data(), L->dqk, L->rope_dim, L->rope_base, double(p), qr.data());
  const int lo = (L->window > 0) ? std::max(0, p - L->window + 1) : 0;
  const int n = p - lo + 1;
  const bool has_sink = L->sink != nullptr;
  const double sink = has_sink ? double(L->sink[h]) : 0.0;

  if (!online) {
    std::vector<double> z(n);
    double M = has_sink ? sink : -INFINITY;
    for (int t = 0; t < n; ++t) {
      if (!fetch_key(C, s, lo + t, g, k.data(), nullptr)) return -2;
      double dot = 0.0;
      for (int d = 0; d < L->dqk; ++d) dot += qr[d] * k[d];
      z[t] = L->softmax_scale * dot;
      if (z[t] > M) M = z[t];
    }
    double Z = has_sink ? std::exp(sink - M) : 0.0;
    std::vector<double> acc(L->dv, 0.0);
    for (int t = 0; t < n; ++t) {
      if (!fetch_key(C, s, lo + t, g, nullptr, v.data())) return -2;
      const double w = std::exp(z[t] - M);
      Z += w;
      for (int d = 0; d < L->dv; ++d) acc[d] += w * v[d];
    }
    for (int d = 0; d < L->dv; ++d) out[d] = L->v_scale * acc[d] / Z;
    *lse = M + std::log(Z);
    return 0;
  }
  // streaming form: running max m, running denominator l, running numerator acc
  double m = has_sink ? sink : -INFINITY;
  double l = has_sink ? 1.0 : 0.0;
  std::vector<double> acc(L->dv, 0.0);
  for (int t = 0; t < n; ++t) {
    if (!fetch_key(C, s, lo + t, g, k.data(), v.data())) return -2;
    double dot = 0.0;
    for (int d = 0; d < L->dqk; ++d) dot += qr[d] * k[d];
    const double z = L->softmax_scale * dot;
    const double m_new = z > m ? z : m;
    const double alpha = (m == -INFINITY) ? 0.0 : std::exp(m - m_new);
    const double w = std::exp(z - m_new);
    l = l * alpha + w;
    for (int d = 0; d < L->dv; ++d) acc[d] = acc[d] * alpha + w * v[d];
    m = m_new;
  }
  for (int d = 0; d < L->dv; ++d) out[d] = L->v_scale * acc[d] / l;
  *lse = m + std::log(l);
  return 0;
}

}  // namespace

extern "C" {

// Evaluates the selected query rows (sel_seq[i], sel_row[i] = row within the
// sequence) for all heads.  out: [n_sel, hq, dv] double; lse: [n_sel, hq] double.
// Returns 0, -1 for a bad argument, -2 when a needed key position is held nowhere.
int oracle_attention(const oracle_layer* L, const uint16_t* q, int n_sel, const int32_t* sel_seq,
                     const int32_t* sel_row, double* out, double* lse, int nthreads, int online) {
  if (!L || !q || n_sel < 0 || L->hq <= 0 || L->hkv <= 0 || L->hq % L->hkv || L->rope_dim % 2 ||
      L->rope_dim > L->dqk)
    return -1;
  for (int i = 0; i < n_sel; ++i) {
    if (sel_seq[i] < 0 || sel_seq[i] >= L->num_seqs) return -1;
    if (sel_row[i] < 0 || sel_row[i] >= L->q_len[sel_seq[i]]) return -1;
  }
  Ctx C;
  C.L = L;
  C.q = q;
  prepare(C);
  const long total = long(n_sel) * L->hq;
  std::atomic<long> next(0);
  std::atomic<int> err(0);
  auto worker = [&]() {
    for (;;) {
      const long w = next.fetch_add(1);
      if (w >= total) break;
      const int i = int(w / L->hq), h = int(w % L->hq);
      const int rc = one_row(C, sel_seq[i], sel_row[i], h, online, out + (size_t(i) * L->hq + h) * L->dv,
                             lse + size_t(i) * L->hq + h);
      if (rc) err.store(rc);
    }
  };
  if (nthreads < 1) nthreads = 1;
  std::vector<std::thread> th;
  for (int t = 1; t < nthreads; ++t) th.emplace_back(worker);
  worker();
  for (auto& t : th) t.join();
  return err.load();
}

// Expected cache contents after appending new tokens: the key rotated at its
// position (double), the value unchanged (double).  k_out: [n, hkv, dqk], v_out: [n, hkv, dv].
int oracle_kv_append(int n, int hkv, int dqk, int dv, int rope_dim, double rope_base, const uint16_t* k_new,
                     const uint16_t* v_new, const int32_t* pos, double* k_out, double* v_out) {
  std::vector<double> x(dqk);
  for (int t = 0; t < n; ++t)
    for (int g = 0; g < hkv; ++g) {
      const uint16_t* kp = k_new + (size_t(t) * hkv + g) * dqk;
      for (int i = 0; i < dqk; ++i) x[i] = bf16_to_double(kp[i]);
      oracle_rope(x.data(), dqk, rope_dim, rope_base, double(pos[t]), k_out + (size_t(t) * hkv + g) * dqk);
      const uint16_t* vp = v_new + (size_t(t) * hkv + g) * dv;
      for (int i = 0; i < dv; ++i) v_out[(size_t(t) * hkv + g) * dv + i] = bf16_to_double(vp[i]);
    }
  return 0;
}

}  // extern "C"
