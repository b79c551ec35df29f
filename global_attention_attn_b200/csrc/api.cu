// C-ABI entry points of libmimoattn: host-side validation, TMA descriptors,
// workspace carving and kernel dispatch.  See include/mimoattn.h for the
// contract of each call.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <climits>
#include <cstring>
#include <mutex>

#include "../../include/mimoattn.h"
#include "internal.h"

namespace mimo {

__device__ unsigned g_status_word;

// Split-KV partials of mimo_attn_decode_noalloc.  Device code never names it: host code
// passes the per-device address that dev_state() looks up.
static __device__ __align__(256) unsigned char g_decode_scratch[MIMO_DECODE_NOALLOC_MAX_BYTES];

namespace {

thread_local char g_err[512] = "";

int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return code;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

#define REQUIRE_PTR(p, name)                                                                        \
  do {                                                                                              \
    if ((p) == nullptr) return fail(MIMO_ERR_INVALID_ARG, "%s: %s is NULL", fn, name);             \
    if (!aligned16(p)) return fail(MIMO_ERR_INVALID_ARG, "%s: %s is not 16-byte aligned", fn, name); \
  } while (0)

int check_layer(const char* fn, const mimo_layer& L) {
  if (L.num_q_heads != kHq || L.head_dim_qk != kDqk || L.head_dim_v != kDv || L.rope_dim != kRope)
    return fail(MIMO_ERR_UNSUPPORTED, "%s: only 64 query heads, head dims 192/128 and rope_dim 64 are supported", fn);
  if (L.num_kv_heads != 8 && L.num_kv_heads != 4)
    return fail(MIMO_ERR_UNSUPPORTED, "%s: num_kv_heads must be 8 or 4 (got %d)", fn, L.num_kv_heads);
  if (!(L.rope_base > 0.0) || !std::isfinite(L.rope_base))
    return fail(MIMO_ERR_INVALID_ARG, "%s: rope_base must be a finite positive number", fn);
  if (!(L.softmax_scale > 0.f) || !std::isfinite(L.softmax_scale))
    return fail(MIMO_ERR_INVALID_ARG, "%s: softmax_scale must be finite and positive", fn);
  if (!std::isfinite(L.v_scale)) return fail(MIMO_ERR_INVALID_ARG, "%s: v_scale must be finite", fn);
  if (L.window < 0) return fail(MIMO_ERR_INVALID_ARG, "%s: window must be >= 0", fn);
  if (L.sink && (reinterpret_cast<uintptr_t>(L.sink) & 3))
    return fail(MIMO_ERR_INVALID_ARG, "%s: sink is not 4-byte aligned", fn);
  return MIMO_OK;
}

// Every bounded wait of the kernels gives up after this long by default.
constexpr unsigned long long kWaitNs = 2000000000ull;

RopeFreqs make_freqs(double base) {
  RopeFreqs f;
  for (int j = 0; j < kHalf; ++j) f.inv_freq[j] = std::pow(base, -2.0 * double(j) / double(kRope));
  return f;
}

// Id of the calling thread's current CUDA context (0 if none), through the driver entry
// points the runtime exposes: a context that was destroyed and re-created (a device reset)
// gets a new id, and its module globals new addresses.
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);
unsigned long long current_ctx_id() {
  static CtxGetCurrentFn get_cur = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_cur = reinterpret_cast<CtxGetCurrentFn>(f);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(f);
  });
  CUcontext c = nullptr;
  unsigned long long id = 0;
  if (!get_cur || !get_id || get_cur(&c) != CUDA_SUCCESS || !c || get_id(c, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Per-device state: addresses of the status word and of the no-alloc decode scratch in
// this device's copy of the module, the SM count, and the context they belong to.  Looked
// up on the first call on a device (with that device current) and again whenever the
// current context is not the one they were looked up in.
struct DevState {
  unsigned* status = nullptr;
  void* scratch = nullptr;
  int sms = 0;
  unsigned long long ctx = 0;
};
std::mutex g_mu;
DevState g_dev[64];

int dev_state(const char* fn, DevState* out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(MIMO_ERR_CUDA, "%s: cudaGetDevice: %s", fn, cudaGetErrorString(e));
  if (dev < 0 || dev >= 64) return fail(MIMO_ERR_CUDA, "%s: device index %d out of range", fn, dev);
  std::lock_guard<std::mutex> lk(g_mu);
  DevState& d = g_dev[dev];
  if (!d.status || d.ctx != current_ctx_id()) {
    // cudaGetSymbolAddress makes the device's primary context current (creating it if
    // needed), so the context id is read after it.
    void* st = nullptr;
    void* sc = nullptr;
    e = cudaGetSymbolAddress(&st, g_status_word);
    if (e != cudaSuccess || !st)
      return fail(MIMO_ERR_CUDA, "%s: cudaGetSymbolAddress (status word): %s", fn, cudaGetErrorString(e));
    e = cudaGetSymbolAddress(&sc, g_decode_scratch);
    if (e != cudaSuccess || !sc)
      return fail(MIMO_ERR_CUDA, "%s: cudaGetSymbolAddress (decode scratch): %s", fn, cudaGetErrorString(e));
    int sms = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return fail(MIMO_ERR_CUDA, "%s: cudaDeviceGetAttribute: %s", fn, cudaGetErrorString(e));
    d.status = static_cast<unsigned*>(st);
    d.scratch = sc;
    d.sms = sms;
    d.ctx = current_ctx_id();
  }
  *out = d;
  return MIMO_OK;
}

// Slots per sequence of a ring cache: 0 means the default; else a multiple of the 16-key
// tile in [128, 512].
int ring_slots_of(const char* fn, int v, int* out) {
  if (v == 0) v = MIMO_RING_SLOTS_DEFAULT;
  if (v < MIMO_RING_SLOTS_DEFAULT || v > MIMO_RING_SLOTS_MAX || v % 16)
    return fail(MIMO_ERR_INVALID_ARG, "%s: ring_slots must be 0 (128) or a multiple of 16 in 128..512 (got %d)", fn,
                v);
  *out = v;
  return MIMO_OK;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

int get_encoder(const char* fn, EncodeTiledFn* out) {
  static EncodeTiledFn enc = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      enc = reinterpret_cast<EncodeTiledFn>(f);
  });
  if (!enc) return fail(MIMO_ERR_CUDA, "%s: cuTensorMapEncodeTiled is not available", fn);
  *out = enc;
  return MIMO_OK;
}

// 3-D bf16 tensor [rows, heads, dim] (dim innermost) with box {64, box_h, box_rows},
// 128-byte swizzle, zero fill out of bounds.
int check_cache_dtype(const char* fn, int dtype, const float* kdq, const float* vdq) {
  if (dtype != MIMO_DTYPE_BF16 && dtype != MIMO_DTYPE_FP8_E4M3)
    return fail(MIMO_ERR_INVALID_ARG, "%s: unknown cache_dtype %d", fn, dtype);
  if (dtype == MIMO_DTYPE_FP8_E4M3) {
    if (!kdq || !vdq) return fail(MIMO_ERR_INVALID_ARG, "%s: an E4M3 cache needs k_dequant and v_dequant", fn);
    if ((reinterpret_cast<uintptr_t>(kdq) | reinterpret_cast<uintptr_t>(vdq)) & 3)
      return fail(MIMO_ERR_INVALID_ARG, "%s: k_dequant / v_dequant are not 4-byte aligned", fn);
  }
  return MIMO_OK;
}

// 3-D map [rows, heads, dim] with boxes of 64 elements x box_h heads x box_rows rows:
// bf16 with the 128-byte swizzle, or (fp8) one-byte elements with the 64-byte swizzle.
int make_map(const char* fn, EncodeTiledFn enc, CUtensorMap* m, const void* base, long rows, int heads, int dim,
             int box_h, int box_rows, bool fp8 = false) {
  const cuuint64_t es = fp8 ? 1 : 2;
  cuuint64_t gdim[3] = {cuuint64_t(dim), cuuint64_t(heads), cuuint64_t(rows < 1 ? 1 : rows)};
  cuuint64_t gstride[2] = {cuuint64_t(dim) * es, cuuint64_t(dim) * es * heads};
  cuuint32_t box[3] = {64, cuuint32_t(box_h), cuuint32_t(box_rows)};
  cuuint32_t estride[3] = {1, 1, 1};
  CUresult r = enc(m, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                   const_cast<void*>(base), gdim, gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   fp8 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MIMO_ERR_CUDA, "%s: cuTensorMapEncodeTiled failed (%d)", fn, int(r));
  return MIMO_OK;
}

size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

// Keys a decode unit range covers at most: the window of the earliest of q_len query rows
// reaches q_len - 1 keys further back than the last row's.
int decode_unit_keys(int max_seq_len, int window, int q_len) {
  if (window <= 0) return max_seq_len;
  const long w = long(window) + q_len - 1;
  return w < max_seq_len ? int(w) : max_seq_len;
}

// Keys per decode split (a multiple of the kernel's 16-key tile).
int decode_split_len(int unit_keys) {
  if (unit_keys <= 256) return 256;
  if (unit_keys <= 8192) return 512;
  return 1024;
}

// Split-KV partials of a decode call: (batch * q_len) query rows x 64 heads x splits.
size_t decode_workspace(int batch, int q_len, int max_seq_len, int window) {
  if (batch <= 0 || max_seq_len <= 0 || q_len <= 0) return 0;
  const int n = decode_unit_keys(max_seq_len, window, q_len);
  const int split = decode_split_len(n);
  const int ns = (n + split - 1) / split;
  if (ns <= 1) return 0;
  const size_t rows = size_t(batch) * q_len;
  return round256(rows * kHq * ns * kDv * 4) + round256(rows * kHq * ns * 2 * 4);
}

// Draft verification of a global layer on a bf16 paged cache: the q_len rows of a sequence's 16
// heads fill half or all of the tensor-core prefill kernel's 128-row tile, which reads each
// 128-key page once per split for all of them.  Splits are whole pages: the decode's split length
// (a multiple of 128), doubled beyond 8192 keys, where a unit's fixed costs (its query tile, the
// partials written and merged) weigh more than the balance of the last round; never shorter than
// the decode's, so the partials fit its workspace and its combine pass merges them.
int decode_drafts_paged_tc(const char* fn, const mimo_decode_args* a, int q_len, void* stream) {
  DevState d;
  if (int rc = dev_state(fn, &d)) return rc;
  EncodeTiledFn enc;
  if (int rc = get_encoder(fn, &enc)) return rc;
  const int hkv = a->layer.num_kv_heads;
  PrefillParams p;
  std::memset(&p, 0, sizeof(p));
  const long rows = long(a->num_pages) * kPage;
  int rc = make_map(fn, enc, &p.tm_q, a->q, long(a->batch) * q_len, kHq, kDqk, 16, prefill_rows_per_tile(1));
  if (!rc) rc = make_map(fn, enc, &p.tm_k0, a->k_cache, rows, hkv, kDqk, 1, 128);
  if (!rc) rc = make_map(fn, enc, &p.tm_k12, a->k_cache, rows, hkv, kDqk, 1, 128);
  if (!rc) rc = make_map(fn, enc, &p.tm_v, a->v_cache, rows, hkv, kDv, 1, 128);
  if (rc) return rc;
  const int split_len = decode_split_len(a->max_seq_len) * (a->max_seq_len > 8192 ? 2 : 1);
  const int max_splits = (a->max_seq_len + split_len - 1) / split_len;
  p.num_seqs = a->batch;
  p.total_q = a->batch * q_len;
  p.hkv = hkv;
  p.mode = kModePaged;
  p.window = 0;
  p.max_pages = a->max_pages;
  p.num_pages = a->num_pages;
  p.scale_log2 = a->layer.softmax_scale * 1.4426950408889634f;
  p.v_scale = a->layer.v_scale;
  p.sink = a->layer.sink;
  p.out = static_cast<uint16_t*>(a->out);
  p.lse = a->lse;
  p.rope = make_freqs(a->layer.rope_base);
  p.status = d.status;
  p.wait_ns = kWaitNs;
  p.uq = q_len;
  if (max_splits > 1) {
    p.split_tiles = split_len / kPage;
    p.max_splits = max_splits;
    p.ws_o = static_cast<float*>(a->workspace);
    p.ws_ml = reinterpret_cast<float*>(static_cast<char*>(a->workspace) +
                                       round256(size_t(a->batch) * q_len * kHq * max_splits * kDv * 4));
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const long work = long(a->batch) * hkv * max_splits;
  const int grid = int(work < d.sms ? work : d.sms);
  if (a->ev_kernel_begin) {
    cudaError_t e = cudaEventRecord(static_cast<cudaEvent_t>(a->ev_kernel_begin), st);
    if (e != cudaSuccess) return fail(MIMO_ERR_CUDA, "%s: ev_kernel_begin: %s", fn, cudaGetErrorString(e));
  }
  for (int s0 = 0; s0 < a->batch; s0 += kPrefillMaxSeqsPerLaunch) {
    PrefillParams q = p;
    q.seq_base = s0;
    q.num_seqs = a->batch - s0 < kPrefillMaxSeqsPerLaunch ? a->batch - s0 : kPrefillMaxSeqsPerLaunch;
    q.seq_lens = a->seq_lens + s0;
    q.block_table = a->block_table + long(s0) * a->max_pages;
    cudaError_t e = launch_prefill(q, 1, grid, st, false);
    if (e != cudaSuccess) return fail(MIMO_ERR_CUDA, "%s: launch failed: %s", fn, cudaGetErrorString(e));
  }
  if (a->ev_kernel_end) {
    cudaError_t e = cudaEventRecord(static_cast<cudaEvent_t>(a->ev_kernel_end), st);
    if (e != cudaSuccess) return fail(MIMO_ERR_CUDA, "%s: ev_kernel_end: %s", fn, cudaGetErrorString(e));
  }
  if (max_splits > 1) {
    DecodeParams c;
    std::memset(&c, 0, sizeof(c));
    c.batch = a->batch;
    c.hkv = hkv;
    c.group = kHq / hkv;
    c.q_len = q_len;
    c.window = 0;
    c.split_len = split_len;
    c.max_splits = max_splits;
    c.v_scale = a->layer.v_scale;
    c.sink = a->layer.sink;
    c.seq_lens = a->seq_lens;
    c.out = p.out;
    c.lse = a->lse;
    c.ws_o = p.ws_o;
    c.ws_ml = p.ws_ml;
    c.status = d.status;
    cudaError_t e = launch_decode_combine(c, st);
    if (e != cudaSuccess) return fail(MIMO_ERR_CUDA, "%s: combine launch failed: %s", fn, cudaGetErrorString(e));
  }
  return MIMO_OK;
}

}  // namespace
}  // namespace mimo

using namespace mimo;

extern "C" {

const char* mimo_last_error(void) { return g_err; }

const char* mimo_version(void) { return "libmimoattn 0.1 (sm_100a)"; }

int mimo_window_from_left_right(int left, int right, int* window) {
  const char* fn = "mimo_window_from_left_right";
  if (!window) return fail(MIMO_ERR_INVALID_ARG, "%s: window is NULL", fn);
  if (right != 0) return fail(MIMO_ERR_UNSUPPORTED, "%s: right = %d: the layers are causal (right must be 0)", fn, right);
  if (left < -1 || left == INT_MAX)
    return fail(MIMO_ERR_INVALID_ARG, "%s: left must be -1 (unbounded) or in 0..INT_MAX-1 (got %d)", fn, left);
  *window = left + 1;
  return MIMO_OK;
}

size_t mimo_attn_prefill_workspace_size(int num_seqs, int total_q, int total_k, int num_kv_heads, int cache_kind) {
  if (num_seqs < 0 || total_q < 0 || total_k < 0 || num_kv_heads <= 0) return 0;
  if (cache_kind == MIMO_CACHE_PAGED) return 0;
  const size_t cs = round256(size_t(total_q) * kHalf * 8);  // (cos, sin) per query row and frequency
  if (cache_kind == MIMO_CACHE_RING) {
    const size_t rows = size_t(total_k) + 128 * size_t(num_seqs);
    return round256(rows * num_kv_heads * kDqk * 2) + round256(rows * num_kv_heads * kDv * 2) +
           round256(size_t(total_k) * num_kv_heads * kRope * 2) + cs;
  }
  return round256(size_t(total_k) * num_kv_heads * kRope * 2) + cs;
}

size_t mimo_attn_decode_workspace_size(int batch, int max_seq_len, int num_kv_heads, int window) {
  (void)num_kv_heads;
  return decode_workspace(batch, 1, max_seq_len, window);
}

size_t mimo_attn_verify_workspace_size(int batch, int q_len, int max_seq_len, int num_kv_heads, int window) {
  (void)num_kv_heads;
  if (q_len < 1 || q_len > MIMO_MAX_DRAFTS) return 0;
  return decode_workspace(batch, q_len, max_seq_len, window);
}

int mimo_kv_append(const mimo_append_args* a, void* stream) {
  const char* fn = "mimo_kv_append";
  if (!a) return fail(MIMO_ERR_INVALID_ARG, "%s: args is NULL", fn);
  if (a->head_dim_qk != kDqk || a->head_dim_v != kDv || a->rope_dim != kRope)
    return fail(MIMO_ERR_UNSUPPORTED, "%s: only head dims 192/128 and rope_dim 64 are supported", fn);
  if (a->num_kv_heads != 8 && a->num_kv_heads != 4)
    return fail(MIMO_ERR_UNSUPPORTED, "%s: num_kv_heads must be 8 or 4", fn);
  if (!(a->rope_base > 0.0) || !std::isfinite(a->rope_base))
    return fail(MIMO_ERR_INVALID_ARG, "%s: rope_base must be a finite positive number", fn);
  if (a->num_tokens < 0) return fail(MIMO_ERR_INVALID_ARG, "%s: num_tokens must be >= 0", fn);
  if (a->cache_kind != MIMO_CACHE_RING && a->cache_kind != MIMO_CACHE_PAGED)
    return fail(MIMO_ERR_INVALID_ARG, "%s: cache_kind must be MIMO_CACHE_RING or MIMO_CACHE_PAGED", fn);
  if (a->num_seqs <= 0) return fail(MIMO_ERR_INVALID_ARG, "%s: num_seqs must be > 0", fn);
  if (a->num_tokens == 0) return MIMO_OK;
  REQUIRE_PTR(a->k_new, "k_new");
  REQUIRE_PTR(a->v_new, "v_new");
  REQUIRE_PTR(a->pos, "pos");
  REQUIRE_PTR(a->seq_idx, "seq_idx");
  REQUIRE_PTR(a->k_cache, "k_cache");
  REQUIRE_PTR(a->v_cache, "v_cache");
  if (a->cache_kind == MIMO_CACHE_PAGED) {
    REQUIRE_PTR(a->block_table, "block_table");
    if (a->max_pages <= 0 || a->num_pages <= 0)
      return fail(MIMO_ERR_INVALID_ARG, "%s: max_pages and num_pages must be > 0 for a paged cache", fn);
  }
  if (int rc = check_cache_dtype(fn, a->cache_dtype, a->k_dequant, a->v_dequant)) return rc;
  int ring_slots = 0;
  if (int rc = ring_slots_of(fn, a->ring_slots, &ring_slots)) return rc;
  DevState d;
  if (int rc = dev_state(fn, &d)) return rc;
  AppendParams p;
  p.ring_slots = ring_slots;
  p.num_tokens = a->num_tokens;
  p.hkv = a->num_kv_heads;
  p.k_new = static_cast<const uint16_t*>(a->k_new);
  p.v_new = static_cast<const uint16_t*>(a->v_new);
  p.pos = a->pos;
  p.seq_idx = a->seq_idx;
  p.cache_kind = a->cache_kind;
  p.k_cache = static_cast<uint16_t*>(a->k_cache);
  p.v_cache = static_cast<uint16_t*>(a->v_cache);
  p.num_seqs = a->num_seqs;
  p.block_table = a->block_table;
  p.max_pages = a->max_pages;
  p.num_pages = a->num_pages;
  p.fp8 = a->cache_dtype == MIMO_DTYPE_FP8_E4M3;
  p.k_dequant = a->k_dequant;
  p.v_dequant = a->v_dequant;
  p.rope = make_freqs(a->rope_base);
  p.status = d.status;
  cudaError_t e = launch_kv_append(p, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(MIMO_ERR_CUDA, "%s: launch failed: %s", fn, cudaGetErrorString(e));
  return MIMO_OK;
}

int mimo_attn_decode(const mimo_decode_args* a, void* stream) {
  const char* fn = "mimo_attn_decode";
  if (!a) return fail(MIMO_ERR_INVALID_ARG, "%s: args is NULL", fn);
  if (int rc = check_layer(fn, a->layer)) return rc;
  if (a->batch < 0) return fail(MIMO_ERR_INVALID_ARG, "%s: batch must be >= 0", fn);
  if (a->batch == 0) return MIMO_OK;
  if (a->max_seq_len <= 0) return fail(MIMO_ERR_INVALID_ARG, "%s: max_seq_len must be > 0", fn);
  if (a->cache_kind != MIMO_CACHE_RING && a->cache_kind != MIMO_CACHE_PAGED)
    return fail(MIMO_ERR_INVALID_ARG, "%s: cache_kind must be MIMO_CACHE_RING or MIMO_CACHE_PAGED", fn);
  int ring_slots = 0;
  if (int rc = ring_slots_of(fn, a->ring_slots, &ring_slots)) return rc;
  const int q_len = a->q_len == 0 ? 1 : a->q_len;
  if (q_len < 1 || q_len > MIMO_MAX_DRAFTS)
    return fail(MIMO_ERR_INVALID_ARG, "%s: q_len must be 0 or 1 (decode) or at most %d draft tokens (got %d)", fn,
                MIMO_MAX_DRAFTS, a->q_len);
  if (a->cache_kind == MIMO_CACHE_RING && (a->layer.window <= 0 || long(a->layer.window) + q_len - 1 > ring_slots))
    return fail(MIMO_ERR_INVALID_ARG,
                "%s: a ring cache of %d slots holds %d positions: window + q_len - 1 must be in 1..%d (window %d, "
                "q_len %d)",
                fn, ring_slots, ring_slots, ring_slots, a->layer.window, q_len);
  if (a->max_seq_len < q_len) return fail(MIMO_ERR_INVALID_ARG, "%s: max_seq_len is below q_len", fn);
  REQUIRE_PTR(a->q, "q");
  REQUIRE_PTR(a->seq_lens, "seq_lens");
  REQUIRE_PTR(a->k_cache, "k_cache");
  REQUIRE_PTR(a->v_cache, "v_cache");
  REQUIRE_PTR(a->out, "out");
  if (a->lse && (reinterpret_cast<uintptr_t>(a->lse) & 3))
    return fail(MIMO_ERR_INVALID_ARG, "%s: lse is not 4-byte aligned", fn);
  if (a->cache_kind == MIMO_CACHE_PAGED) {
    REQUIRE_PTR(a->block_table, "block_table");
    if (a->max_pages <= 0 || a->num_pages <= 0)
      return fail(MIMO_ERR_INVALID_ARG, "%s: max_pages and num_pages must be > 0 for a paged cache", fn);
    if (long(a->max_pages) * kPage < a->max_seq_len)
      return fail(MIMO_ERR_INVALID_ARG, "%s: max_pages * 128 is below max_seq_len", fn);
  }
  if (int rc = check_cache_dtype(fn, a->cache_dtype, a->k_dequant, a->v_dequant)) return rc;
  const size_t need = decode_workspace(a->batch, q_len, a->max_seq_len, a->layer.window);
  if (need > 0) {
    if (!a->workspace || a->workspace_bytes < need)
      return fail(MIMO_ERR_WORKSPACE, "%s: workspace of %zu bytes required (got %zu)", fn, need,
                  a->workspace ? a->workspace_bytes : size_t(0));
    if (!aligned16(a->workspace)) return fail(MIMO_ERR_INVALID_ARG, "%s: workspace is not 16-byte aligned", fn);
  }
  if (q_len >= 2 && a->cache_kind == MIMO_CACHE_PAGED && a->cache_dtype != MIMO_DTYPE_FP8_E4M3 &&
      a->layer.window <= 0 && a->layer.num_kv_heads == 4)
    return decode_drafts_paged_tc(fn, a, q_len, stream);
  DevState d;
  if (int rc = dev_state(fn, &d)) return rc;
  EncodeTiledFn enc;
  if (int rc = get_encoder(fn, &enc)) return rc;
  DecodeParams p;
  std::memset(&p, 0, sizeof(p));
  {
    const long rows = a->cache_kind == MIMO_CACHE_RING ? long(a->batch) * ring_slots : long(a->num_pages) * kPage;
    const bool fp8 = a->cache_dtype == MIMO_DTYPE_FP8_E4M3;
    // queries [batch * q_len, 64, 192]: a 16-row block is 16 heads of one row (global layers)
    // or 8 heads of two rows (sliding-window layers)
    const int G = kHq / a->layer.num_kv_heads;
    int rc = make_map(fn, enc, &p.tm_q, a->q, long(a->batch) * q_len, kHq, kDqk, G, 16 / G);
    if (!rc) rc = make_map(fn, enc, &p.tm_k, a->k_cache, rows, a->layer.num_kv_heads, kDqk, 1, 16, fp8);
    if (!rc) rc = make_map(fn, enc, &p.tm_v, a->v_cache, rows, a->layer.num_kv_heads, kDv, 1, 16, fp8);
    if (rc) return rc;
  }
  p.batch = a->batch;
  p.hkv = a->layer.num_kv_heads;
  p.group = kHq / p.hkv;
  p.window = a->layer.window;
  p.q_len = q_len;
  {
    int nc = 0;
    decode_rows(q_len, p.group, &p.n_blocks, &nc, &p.n_rp);
  }
  const int n = decode_unit_keys(a->max_seq_len, p.window, q_len);
  p.split_len = decode_split_len(n);
  p.max_splits = (n + p.split_len - 1) / p.split_len;
  if (a->cache_kind == MIMO_CACHE_RING && p.max_splits != 1)  // window + q_len - 1 <= 512 keys: one split
    return fail(MIMO_ERR_INVALID_ARG, "%s: a ring decode takes one split (internal)", fn);
  p.scale_log2 = a->layer.softmax_scale * 1.4426950408889634f;
  p.v_scale = a->layer.v_scale;
  p.sink = a->layer.sink;
  p.q = static_cast<const uint16_t*>(a->q);
  p.seq_lens = a->seq_lens;
  p.cache_kind = a->cache_kind;
  p.ring_slots = ring_slots;
  p.k_cache = static_cast<const uint16_t*>(a->k_cache);
  p.v_cache = static_cast<const uint16_t*>(a->v_cache);
  p.block_table = a->block_table;
  p.max_pages = a->max_pages;
  p.num_pages = a->num_pages;
  p.out = static_cast<uint16_t*>(a->out);
  p.lse = a->lse;
  p.ws_o = need ? static_cast<float*>(a->workspace) : nullptr;
  p.ws_ml = need ? reinterpret_cast<float*>(static_cast<char*>(a->workspace) +
                                            round256(size_t(a->batch) * q_len * kHq * p.max_splits * kDv * 4))
                 : nullptr;
  p.fp8 = a->cache_dtype == MIMO_DTYPE_FP8_E4M3;
  p.k_dequant = a->k_dequant;
  p.v_dequant = a->v_dequant;
  p.rope = make_freqs(a->layer.rope_base);
  p.status = d.status;
  cudaError_t e = launch_decode(p, d.sms, static_cast<cudaStream_t>(stream), a->ev_kernel_begin, a->ev_kernel_end);
  if (e != cudaSuccess) return fail(MIMO_ERR_CUDA, "%s: launch failed: %s", fn, cudaGetErrorString(e));
  return MIMO_OK;
}

}  // extern "C"

namespace mimo {
namespace {


int prefill_impl(const char* fn, const mimo_prefill_args* a, void* stream, unsigned long long wait_ns,
                 int withhold_q) {
  if (!a) return fail(MIMO_ERR_INVALID_ARG, "%s: args is NULL", fn);
  if (int rc = check_layer(fn, a->layer)) return rc;
  if (a->num_seqs <= 0) return fail(MIMO_ERR_INVALID_ARG, "%s: num_seqs must be > 0", fn);
  if (a->total_q < 0 || a->total_k < 0) return fail(MIMO_ERR_INVALID_ARG, "%s: total_q/total_k must be >= 0", fn);
  if (a->cache_kind != MIMO_CACHE_NONE && a->cache_kind != MIMO_CACHE_RING && a->cache_kind != MIMO_CACHE_PAGED)
    return fail(MIMO_ERR_INVALID_ARG, "%s: unknown cache_kind %d", fn, a->cache_kind);
  if (a->total_q == 0) return MIMO_OK;
  REQUIRE_PTR(a->q, "q");
  REQUIRE_PTR(a->out, "out");
  REQUIRE_PTR(a->cu_seqlens_q, "cu_seqlens_q");
  if (a->lse && (reinterpret_cast<uintptr_t>(a->lse) & 3))
    return fail(MIMO_ERR_INVALID_ARG, "%s: lse is not 4-byte aligned", fn);
  const int hkv = a->layer.num_kv_heads;
  int mode, ring_slots = 0;
  if (int rc = ring_slots_of(fn, a->ring_slots, &ring_slots)) return rc;
  if (a->cache_kind == MIMO_CACHE_PAGED) {
    if (a->k || a->v || a->cu_seqlens_k || a->total_k)
      return fail(MIMO_ERR_INVALID_ARG,
                  "%s: with a paged cache all keys come from the cache (append them first); k, v, cu_seqlens_k "
                  "must be NULL and total_k 0",
                  fn);
    REQUIRE_PTR(a->k_cache, "k_cache");
    REQUIRE_PTR(a->v_cache, "v_cache");
    REQUIRE_PTR(a->block_table, "block_table");
    REQUIRE_PTR(a->cache_lens, "cache_lens");
    if (a->max_pages <= 0 || a->num_pages <= 0)
      return fail(MIMO_ERR_INVALID_ARG, "%s: max_pages and num_pages must be > 0 for a paged cache", fn);
    mode = kModePaged;
  } else {
    if (a->total_k == 0) return fail(MIMO_ERR_INVALID_ARG, "%s: total_k must be > 0 without a paged cache", fn);
    REQUIRE_PTR(a->k, "k");
    REQUIRE_PTR(a->v, "v");
    REQUIRE_PTR(a->cu_seqlens_k, "cu_seqlens_k");
    if (a->cache_kind == MIMO_CACHE_RING) {
      if (a->layer.window < 1 || a->layer.window > 129)
        return fail(MIMO_ERR_INVALID_ARG, "%s: a ring cache needs a window of 1..129 keys", fn);
      REQUIRE_PTR(a->k_cache, "k_cache");
      REQUIRE_PTR(a->v_cache, "v_cache");
      REQUIRE_PTR(a->cache_lens, "cache_lens");
      mode = kModeExt;
    } else {
      mode = kModeContig;
    }
  }
  const size_t need = mimo_attn_prefill_workspace_size(a->num_seqs, a->total_q, a->total_k, hkv, a->cache_kind);
  if (need > 0) {
    if (!a->workspace || a->workspace_bytes < need)
      return fail(MIMO_ERR_WORKSPACE, "%s: workspace of %zu bytes required (got %zu)", fn, need,
                  a->workspace ? a->workspace_bytes : size_t(0));
    if (!aligned16(a->workspace)) return fail(MIMO_ERR_INVALID_ARG, "%s: workspace is not 16-byte aligned", fn);
  }
  const int kind = (a->layer.window >= 1 && a->layer.window <= 129 && mode != kModePaged) ? 0 : 1;
  DevState d;
  if (int rc = dev_state(fn, &d)) return rc;
  EncodeTiledFn enc;
  if (int rc = get_encoder(fn, &enc)) return rc;
  const int tile_h = kind == 0 ? 8 : 16;  // query heads stacked in one M tile (one KV group)
  if (kind == 0 && hkv != 8) return fail(MIMO_ERR_UNSUPPORTED, "%s: sliding-window path needs 8 KV heads", fn);
  if (kind == 1 && hkv != 4) return fail(MIMO_ERR_UNSUPPORTED, "%s: global path needs 4 KV heads", fn);
  const int R = prefill_rows_per_tile(kind);
  const int BN = prefill_key_tile(kind);
  PrefillParams p;
  std::memset(&p, 0, sizeof(p));
  int rc = make_map(fn, enc, &p.tm_q, a->q, a->total_q, kHq, kDqk, tile_h, R);
  if (rc) return rc;
  uint16_t* ws_k = static_cast<uint16_t*>(a->workspace);
  uint16_t* ws_v = nullptr;
  uint16_t* ws_rot = nullptr;
  float2* cs_q = nullptr;
  if (mode != kModePaged) {
    const size_t cs_bytes = round256(size_t(a->total_q) * kHalf * 8);
    cs_q = reinterpret_cast<float2*>(static_cast<char*>(a->workspace) + need - cs_bytes);
  }
  if (kind == 0) {
    // 2-D fp32 table [total_q, 64] (cos, sin interleaved per frequency), box {64, 16}, no swizzle
    cuuint64_t gdim[2] = {64, cuuint64_t(a->total_q)};
    cuuint64_t gstride[1] = {64 * 4};
    cuuint32_t box[2] = {64, cuuint32_t(R)};
    cuuint32_t estride[2] = {1, 1};
    CUresult r = enc(&p.tm_cs, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, cs_q, gdim, gstride, box, estride,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(MIMO_ERR_CUDA, "%s: cuTensorMapEncodeTiled (cos/sin table) failed (%d)", fn, int(r));
  }
  if (mode == kModeContig) {
    if ((rc = make_map(fn, enc, &p.tm_k0, ws_k, a->total_k, hkv, kRope, 1, BN))) return rc;
    if ((rc = make_map(fn, enc, &p.tm_k12, a->k, a->total_k, hkv, kDqk, 1, BN))) return rc;
    if ((rc = make_map(fn, enc, &p.tm_v, a->v, a->total_k, hkv, kDv, 1, BN))) return rc;
  } else if (mode == kModeExt) {
    // [halo | new] copy of K, of V, then the rotated dims of the new keys
    const long rows = long(a->total_k) + 128L * a->num_seqs;
    const size_t k_bytes = round256(size_t(rows) * hkv * kDqk * 2), v_bytes = round256(size_t(rows) * hkv * kDv * 2);
    ws_v = reinterpret_cast<uint16_t*>(static_cast<char*>(a->workspace) + k_bytes);
    ws_rot = reinterpret_cast<uint16_t*>(static_cast<char*>(a->workspace) + k_bytes + v_bytes);
    if ((rc = make_map(fn, enc, &p.tm_k0, ws_k, rows, hkv, kDqk, 1, BN))) return rc;
    if ((rc = make_map(fn, enc, &p.tm_k12, ws_k, rows, hkv, kDqk, 1, BN))) return rc;
    if ((rc = make_map(fn, enc, &p.tm_v, ws_v, rows, hkv, kDv, 1, BN))) return rc;
    if ((rc = make_map(fn, enc, &p.tm_k0n, ws_rot, a->total_k, hkv, kRope, 1, BN))) return rc;
    if ((rc = make_map(fn, enc, &p.tm_k12n, a->k, a->total_k, hkv, kDqk, 1, BN))) return rc;
    if ((rc = make_map(fn, enc, &p.tm_vn, a->v, a->total_k, hkv, kDv, 1, BN))) return rc;
  } else {
    const long rows = long(a->num_pages) * kPage;
    if ((rc = make_map(fn, enc, &p.tm_k0, a->k_cache, rows, hkv, kDqk, 1, BN))) return rc;
    if ((rc = make_map(fn, enc, &p.tm_k12, a->k_cache, rows, hkv, kDqk, 1, BN))) return rc;
    if ((rc = make_map(fn, enc, &p.tm_v, a->v_cache, rows, hkv, kDv, 1, BN))) return rc;
  }
  p.num_seqs = a->num_seqs;
  p.seq_base = 0;
  p.total_q = a->total_q;
  p.hkv = hkv;
  p.mode = mode;
  p.window = a->layer.window;
  p.cu_q = a->cu_seqlens_q;
  p.cu_k = a->cu_seqlens_k;
  p.cache_lens = a->cache_lens;
  p.block_table = a->block_table;
  p.max_pages = a->max_pages;
  p.num_pages = a->num_pages;
  p.scale_log2 = a->layer.softmax_scale * 1.4426950408889634f;
  p.v_scale = a->layer.v_scale;
  p.sink = a->layer.sink;
  p.out = static_cast<uint16_t*>(a->out);
  p.lse = a->lse;
  p.rope = make_freqs(a->layer.rope_base);
  p.status = d.status;
  p.wait_ns = wait_ns;
  p.withhold_q = withhold_q;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (mode != kModePaged) {
    RopeKParams r;
    r.num_seqs = a->num_seqs;
    r.total_k = a->total_k;
    r.hkv = hkv;
    r.mode = mode;
    r.cu_k = a->cu_seqlens_k;
    r.cache_lens = a->cache_lens;
    r.k = static_cast<const uint16_t*>(a->k);
    r.v = static_cast<const uint16_t*>(a->v);
    r.ring_k = static_cast<const uint16_t*>(a->k_cache);
    r.ring_v = static_cast<const uint16_t*>(a->v_cache);
    r.ring_slots = ring_slots;
    r.ws_k = ws_k;
    r.ws_v = ws_v;
    r.ws_rot = ws_rot;
    r.total_q = kind == 0 ? a->total_q : 0;
    r.cu_q = a->cu_seqlens_q;
    r.cs_q = cs_q;
    r.rope = p.rope;
    r.status = d.status;
    cudaError_t e = launch_rope_k(r, st);
    if (e != cudaSuccess) return fail(MIMO_ERR_CUDA, "%s: key pre-pass launch failed: %s", fn, cudaGetErrorString(e));
  }
  // upper bound of M tiles: ceil(total_q / R) + num_seqs partial tiles, times KV heads
  const long work = (long(a->total_q) / R + a->num_seqs + 1) * hkv;
  const int grid = int(work < d.sms ? work : d.sms);
  // one launch per group of at most 256 sequences (the kernel keeps a per-sequence table in shared memory)
  if (a->ev_kernel_begin) {
    cudaError_t e = cudaEventRecord(static_cast<cudaEvent_t>(a->ev_kernel_begin), st);
    if (e != cudaSuccess) return fail(MIMO_ERR_CUDA, "%s: ev_kernel_begin: %s", fn, cudaGetErrorString(e));
  }
  for (int s0 = 0; s0 < a->num_seqs; s0 += kPrefillMaxSeqsPerLaunch) {
    PrefillParams q = p;
    q.seq_base = s0;
    q.num_seqs = a->num_seqs - s0 < kPrefillMaxSeqsPerLaunch ? a->num_seqs - s0 : kPrefillMaxSeqsPerLaunch;
    q.cu_q = a->cu_seqlens_q + s0;
    q.cu_k = a->cu_seqlens_k ? a->cu_seqlens_k + s0 : nullptr;
    q.cache_lens = a->cache_lens ? a->cache_lens + s0 : nullptr;
    q.block_table = a->block_table ? a->block_table + long(s0) * a->max_pages : nullptr;
    // overlap the first launch with the key pre-pass, unless the caller times the kernel alone
    const bool pdl = s0 == 0 && mode != kModePaged && !a->ev_kernel_begin && !a->ev_kernel_end;
    cudaError_t e = launch_prefill(q, kind, grid, st, pdl);
    if (e != cudaSuccess) return fail(MIMO_ERR_CUDA, "%s: launch failed: %s", fn, cudaGetErrorString(e));
  }
  if (a->ev_kernel_end) {
    cudaError_t e = cudaEventRecord(static_cast<cudaEvent_t>(a->ev_kernel_end), st);
    if (e != cudaSuccess) return fail(MIMO_ERR_CUDA, "%s: ev_kernel_end: %s", fn, cudaGetErrorString(e));
  }
  return MIMO_OK;
}

}  // namespace
}  // namespace mimo

extern "C" {

int mimo_attn_prefill(const mimo_prefill_args* a, void* stream) {
  return prefill_impl("mimo_attn_prefill", a, stream, kWaitNs, 0);
}

int mimo_attn_prefill_stall_test(const mimo_prefill_args* a, void* stream, unsigned long long wait_limit_ns) {
  const char* fn = "mimo_attn_prefill_stall_test";
  if (wait_limit_ns < 1000000ull || wait_limit_ns > 10000000000ull)
    return fail(MIMO_ERR_INVALID_ARG, "%s: wait_limit_ns must be in 1e6..1e10 (got %llu)", fn, wait_limit_ns);
  return prefill_impl(fn, a, stream, wait_limit_ns, 1);
}

}  // extern "C"

extern "C" {

int mimo_attn_decode_noalloc(const mimo_decode_args* a, void* stream) {
  const char* fn = "mimo_attn_decode_noalloc";
  if (!a) return fail(MIMO_ERR_INVALID_ARG, "%s: args is NULL", fn);
  if (a->batch > 0 && a->max_seq_len > 0) {
    const size_t need = decode_workspace(a->batch, a->q_len == 0 ? 1 : a->q_len, a->max_seq_len, a->layer.window);
    if (need > MIMO_DECODE_NOALLOC_MAX_BYTES)
      return fail(MIMO_ERR_WORKSPACE,
                  "%s: batch %d x max_seq_len %d needs %zu bytes of split-KV partials; the library's static "
                  "scratch holds %u (use mimo_attn_decode with a caller workspace)",
                  fn, a->batch, a->max_seq_len, need, unsigned(MIMO_DECODE_NOALLOC_MAX_BYTES));
  }
  mimo_decode_args b = *a;
  b.workspace = nullptr;
  b.workspace_bytes = 0;
  if (a->batch > 0) {
    // this device's copy of the static array (in host code its name is only a stand-in)
    DevState d;
    if (int rc = dev_state(fn, &d)) return rc;
    b.workspace = d.scratch;
    b.workspace_bytes = MIMO_DECODE_NOALLOC_MAX_BYTES;
  }
  return mimo_attn_decode(&b, stream);
}

int mimo_status_poll(uint32_t* status) {
  const char* fn = "mimo_status_poll";
  if (!status) return fail(MIMO_ERR_INVALID_ARG, "%s: status is NULL", fn);
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return fail(MIMO_ERR_CUDA, "%s: %s", fn, cudaGetErrorString(e));
  unsigned v = 0;
  e = cudaMemcpyFromSymbol(&v, g_status_word, sizeof(v));
  if (e != cudaSuccess) return fail(MIMO_ERR_CUDA, "%s: %s", fn, cudaGetErrorString(e));
  const unsigned zero = 0;
  e = cudaMemcpyToSymbol(g_status_word, &zero, sizeof(zero));
  if (e != cudaSuccess) return fail(MIMO_ERR_CUDA, "%s: %s", fn, cudaGetErrorString(e));
  *status = v;
  if (v & MIMO_STATUS_TIMEOUT) return fail(MIMO_ERR_TIMEOUT, "%s: a device wait gave up (status 0x%x)", fn, v);
  return MIMO_OK;
}

}  // extern "C"
