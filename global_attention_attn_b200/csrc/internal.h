// Internal launch interfaces shared by the host API (api.cu) and the kernel
// translation units.  Not part of the public C ABI.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace mimo {

constexpr int kHq = 64;
constexpr int kDqk = 192;
constexpr int kDv = 128;
constexpr int kRope = 64;
constexpr int kHalf = kRope / 2;
constexpr int kPage = 128;  // positions per page (and the default ring slots)

// Rotary frequencies base^(-2j/64), j = 0..31, evaluated on the host in float64.
struct RopeFreqs {
  double inv_freq[kHalf];
};

struct AppendParams {
  int num_tokens, hkv;
  const uint16_t* k_new;
  const uint16_t* v_new;
  const int32_t* pos;
  const int32_t* seq_idx;
  int cache_kind;
  uint16_t* k_cache;
  uint16_t* v_cache;
  int num_seqs;
  int ring_slots;            // ring: slots per sequence
  const int32_t* block_table;
  int max_pages, num_pages;
  int fp8;                   // cache rows hold E4M3 bytes (quantised by 1 / k_dequant[g], 1 / v_dequant[g])
  const float* k_dequant;
  const float* v_dequant;
  RopeFreqs rope;
  unsigned* status;
};

struct DecodeParams {
  CUtensorMap tm_q;  // queries [batch * q_len, 64, 192], box {64, group, 16 / group}
  CUtensorMap tm_k;  // key cache rows [rows, Hkv, 192], box {64, 1, 16}
  CUtensorMap tm_v;  // value cache rows [rows, Hkv, 128], box {64, 1, 16}
  int batch, hkv, group;  // group = 64 / hkv
  int q_len;              // query rows per sequence: 1 (decode) or 2..8 draft tokens
  int n_blocks, n_rp;     // 16-row blocks of a (sequence, KV head) unit's rows; row parts of a unit
  int window;
  int split_len, max_splits;
  float scale_log2;  // softmax_scale * log2(e)
  float v_scale;
  const float* sink;
  const uint16_t* q;
  const int32_t* seq_lens;
  int cache_kind;
  int ring_slots;  // ring: slots per sequence (a multiple of the 16-key tile)
  const uint16_t* k_cache;
  const uint16_t* v_cache;
  const int32_t* block_table;
  int max_pages, num_pages;
  uint16_t* out;
  float* lse;
  float* ws_o;   // [batch * q_len, 64, max_splits, 128]
  float* ws_ml;  // [batch * q_len, 64, max_splits, 2]
  int fp8;                   // E4M3 cache rows with per-KV-head dequantisation scales
  const float* k_dequant;
  const float* v_dequant;
  RopeFreqs rope;
  unsigned* status;
};

// Key source modes of the prefill kernel.
enum PrefillMode : int {
  kModeContig = 0,  // dims 0..63 from the rotated workspace copy, 64..191 from k, v from v
  kModeExt = 1,     // ring-cache chunk: tiles whose window reaches before the chunk read the
                    // workspace copy [ring halo | first kExtFullRows new keys]; the others read
                    // as kModeContig
  kModePaged = 2,   // everything from the paged cache
};
// New keys of a ring-cache chunk copied whole next to the halo: a 144-key window that starts
// before the chunk ends at most 143 rows into it.
constexpr int kExtFullRows = 144;

struct PrefillParams {
  CUtensorMap tm_q;    // q [total_q, 64, 192], box {64, G, 128/G}
  CUtensorMap tm_k0;   // key dims 0..63 source, box {64, 1, BN}
  CUtensorMap tm_k12;  // key dims 64..191 source (x = 64, 128), box {64, 1, BN}
  CUtensorMap tm_v;    // value source (x = 0, 64), box {64, 1, BN}
  CUtensorMap tm_cs;   // per-query-row cos/sin table [total_q, 64] fp32, box {64, 16} (sliding window)
  // ring-cache chunks (kModeExt): sources of the tiles whose window starts at or after the
  // chunk's first position: rotated dims 0..63 of the new keys, k, v (as kModeContig)
  CUtensorMap tm_k0n, tm_k12n, tm_vn;
  int num_seqs, total_q, hkv, mode, window;
  int seq_base;  // index of this launch's first sequence in the whole batch (launches take <= 256)
  const int32_t* cu_q;
  const int32_t* cu_k;
  const int32_t* cache_lens;
  const int32_t* block_table;
  int max_pages, num_pages;
  float scale_log2;
  float v_scale;
  const float* sink;
  uint16_t* out;
  float* lse;
  RopeFreqs rope;
  unsigned* status;
  unsigned long long wait_ns;  // limit of every bounded wait in the kernel
  int withhold_q;              // failure-detection test: the producer never loads a query tile
  // Draft verification on a paged cache (global kernel only): with cu_q null, sequence s holds
  // the uq query rows (seq_base + s) * uq + i at positions seq_lens[s] - uq + i, i < uq <= 8.
  int uq;
  const int32_t* seq_lens;
  // Split-KV (with uq): split i of a sequence takes key tiles [i * split_tiles, (i + 1) *
  // split_tiles); each split writes its unnormalised O and (running max in log2 units, sum)
  // to ws_o [rows, 64, max_splits, 128] / ws_ml [rows, 64, max_splits, 2] for the decode's
  // combine pass, which adds the sink.  split_tiles 0: one split, final rows written.
  int split_tiles, max_splits;
  float* ws_o;
  float* ws_ml;
};

// Pre-pass of the prefill: rotated key copies into the workspace.
struct RopeKParams {
  int num_seqs, total_k, hkv, mode;
  const int32_t* cu_k;
  const int32_t* cache_lens;
  const uint16_t* k;
  const uint16_t* v;
  const uint16_t* ring_k;  // ext mode: [num_seqs, ring_slots, hkv, D]
  const uint16_t* ring_v;
  int ring_slots;
  uint16_t* ws_k;  // contig: [total_k, hkv, 64]; ext: [total_k + 128*B, hkv, 192]
  uint16_t* ws_v;  // ext: [total_k + 128*B, hkv, 128]
  uint16_t* ws_rot;  // ext: rotated dims 0..63 of the new keys [total_k, hkv, 64]
  // per-query-row (cos, sin) of the 32 rotary frequencies, or null
  int total_q;
  const int32_t* cu_q;
  float2* cs_q;    // [total_q, 32]
  RopeFreqs rope;
  unsigned* status;
};

cudaError_t launch_kv_append(const AppendParams& p, cudaStream_t s);
// ev_begin / ev_end: optional cudaEvent_t recorded around the decode kernel (not the combine)
cudaError_t launch_decode(const DecodeParams& p, int sms, cudaStream_t s, void* ev_begin, void* ev_end);
// The combine pass alone: merges p.max_splits partials per (query row, head) of ws_o / ws_ml.
cudaError_t launch_decode_combine(const DecodeParams& p, cudaStream_t s);
// Row blocks of a decode unit (q_len rows of `group` heads), consumer warps per producer and
// row parts per unit.
void decode_rows(int q_len, int group, int* n_blocks, int* nc, int* n_rp);
cudaError_t launch_rope_k(const RopeKParams& p, cudaStream_t s);
// kind 0: sliding window (G=8 heads x 16 rows, one 144-key tile); kind 1: global (G=16 x 8 rows, 128-key tiles)
// pdl: launch with programmatic stream serialization (the kernel's prologue overlaps the key
// pre-pass launched just before it; its producers wait for the pre-pass before loading)
cudaError_t launch_prefill(const PrefillParams& p, int kind, int grid, cudaStream_t s, bool pdl);
int prefill_rows_per_tile(int kind);
constexpr int kPrefillMaxSeqsPerLaunch = 256;
int prefill_key_tile(int kind);

}  // namespace mimo
