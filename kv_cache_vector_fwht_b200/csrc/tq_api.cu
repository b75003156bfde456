// C ABI of libtq (include/tq.h): argument checks on the host, then kernel launches.
#include <cstdlib>
#include <cstring>
#include <new>

#include "tq_internal.h"

namespace tq {

int sm_count(int device) {
  static int cached[64] = {0};
  if (device < 0 || device >= 64) return 148;
  if (cached[device] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, device) != cudaSuccess || n <= 0)
      n = 148;
    cached[device] = n;
  }
  return cached[device];
}

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int elem_size(int dtype) {
  return dtype == TQ_F32 ? 4 : (dtype == TQ_BF16 || dtype == TQ_F16) ? 2 : 0;
}

tq_status check_rows(const void* x, int dtype, int64_t n_rows, int64_t ld) {
  if (n_rows < 0) return TQ_EINVAL;
  if (dtype != TQ_F32 && dtype != TQ_BF16) return TQ_EUNSUPPORTED;
  if (ld < kD || (ld * elem_size(dtype)) % 16 != 0) return TQ_EINVAL;
  if (n_rows > 0 && (x == nullptr || !aligned16(x))) return TQ_EINVAL;
  return TQ_OK;
}

tq_status check_key_planes(const tq_quantizer* q, const tq_key_planes& p) {
  if (!p.idx || !p.norms) return TQ_EINVAL;
  if (!aligned16(p.idx) || (reinterpret_cast<uintptr_t>(p.norms) & 3u)) return TQ_EINVAL;
  if (q->mode == TQ_MODE_PROD) {
    if (!p.signs || !aligned16(p.signs)) return TQ_EINVAL;
  }
  return TQ_OK;
}

tq_status check_cache(const tq_quantizer* q, const tq_kv_cache* c) {
  if (!c) return TQ_EINVAL;
  if (c->batch <= 0 || c->n_kv_heads <= 0 || c->capacity <= 0 || c->capacity % 16) return TQ_EINVAL;
  if (c->d != kD) return TQ_EUNSUPPORTED;
  if (!c->len_dev || !c->len_host) return TQ_EINVAL;
  if (check_key_planes(q, c->keys) != TQ_OK) return TQ_EINVAL;
  if (!aligned16(c->keys.norms)) return TQ_EINVAL;
  if (c->value_bits != 0) {
    if (c->value_bits != 2 && c->value_bits != 4) return TQ_EUNSUPPORTED;
    if (c->value_group != 32) return TQ_EUNSUPPORTED;
    if (!c->values.q || !c->values.params || !aligned16(c->values.q) || !aligned16(c->values.params))
      return TQ_EINVAL;
  }
  for (int b = 0; b < c->batch; ++b)
    if (c->len_host[b] < 0 || c->len_host[b] > c->capacity) return TQ_EINVAL;
  return TQ_OK;
}

}  // namespace
}  // namespace tq

using namespace tq;

extern "C" {

int tq_abi_version(void) { return TQ_ABI_VERSION; }

tq_status tq_sync_status(void* stream) {
  return take_device_error(static_cast<cudaStream_t>(stream));
}

tq_status tq_selftest_bounded_wait(uint32_t limit_us, void* stream) {
  if (limit_us == 0 || limit_us > 2000000u) return TQ_EINVAL;
  return launch_selftest_wait(limit_us, static_cast<cudaStream_t>(stream));
}

const char* tq_status_string(tq_status s) {
  switch (s) {
    case TQ_OK: return "ok";
    case TQ_EINVAL: return "invalid argument";
    case TQ_EUNSUPPORTED: return "unsupported configuration";
    case TQ_ECAPACITY: return "cache capacity exceeded";
    case TQ_ENOMEM: return "out of memory";
    case TQ_ECUDA: return "CUDA error";
    case TQ_ETIMEOUT: return "device wait timed out";
    case TQ_ETOOLARGE: return "problem exceeds the built-in decode scratch";
  }
  return "unknown status";
}

tq_status tq_host_tables(int d, int bits, int mode, uint64_t seed, const int32_t* outliers,
                         int n_outlier, double* centroids, double* thresholds, int8_t* signs,
                         int32_t* channels, uint16_t* s_rot_fp16) {
  HostTables* t = new (std::nothrow) HostTables;
  if (!t) return TQ_ENOMEM;
  tq_key_layout_t lay;
  const tq_status st = build_host_tables(d, bits, mode, seed, outliers, n_outlier, t, &lay);
  if (st == TQ_OK) {
    if (centroids) std::memcpy(centroids, t->cent, sizeof(t->cent));
    if (thresholds) std::memcpy(thresholds, t->thr, sizeof(t->thr));
    if (signs) std::memcpy(signs, t->signs, sizeof(t->signs));
    if (channels) std::memcpy(channels, t->chan, sizeof(t->chan));
    if (s_rot_fp16 && mode == TQ_MODE_PROD) std::memcpy(s_rot_fp16, t->s_rot, sizeof(t->s_rot));
  }
  delete t;
  return st;
}

namespace {
// Store schedule of the grouped kernel's gather (DevTables::gsched). Lane l stores natural
// channel c = 4l + i to chain position pos[c], a 2-byte slot in bank (pos[c] / 2) mod 32 of a
// row. Lanes x banks with an edge per (l, i) is a 4-regular bipartite multigraph (each bank
// holds chain positions 2b, 2b + 1, 2b + 64, 2b + 65), so it splits into 4 perfect matchings
// (Koenig); each round takes one, found by augmenting paths (Kuhn), and removes it.
bool gather_augment(int l, const int (&bank)[32][4], const bool (&used)[32][4], bool (&seen)[32],
                    int (&lane_of_bank)[32], int (&opt_of_lane)[32]) {
  for (int i = 0; i < 4; ++i) {
    if (used[l][i]) continue;
    const int b = bank[l][i];
    if (seen[b]) continue;
    seen[b] = true;
    if (lane_of_bank[b] < 0 ||
        gather_augment(lane_of_bank[b], bank, used, seen, lane_of_bank, opt_of_lane)) {
      lane_of_bank[b] = l;
      opt_of_lane[l] = i;
      return true;
    }
  }
  return false;
}

void gather_schedule(const int32_t (&chan)[tq::kD], uint8_t (&sched)[32][4]) {
  int pos[tq::kD];
  for (int p = 0; p < tq::kD; ++p) pos[chan[p]] = p;
  int bank[32][4];
  for (int l = 0; l < 32; ++l)
    for (int i = 0; i < 4; ++i) bank[l][i] = (pos[4 * l + i] >> 1) & 31;
  bool used[32][4] = {};
  for (int k = 0; k < 4; ++k) {
    int lane_of_bank[32], opt_of_lane[32];
    for (int j = 0; j < 32; ++j) lane_of_bank[j] = opt_of_lane[j] = -1;
    for (int l = 0; l < 32; ++l) {
      bool seen[32] = {};
      gather_augment(l, bank, used, seen, lane_of_bank, opt_of_lane);
    }
    for (int l = 0; l < 32; ++l) {
      int i = opt_of_lane[l];
      if (i < 0)  // cannot happen for a regular multigraph; any unused channel stays correct
        for (i = 0; used[l][i]; ++i) {}
      used[l][i] = true;
      sched[l][k] = static_cast<uint8_t>(i);
    }
  }
}
}  // namespace

static tq_status build_quantizer(int d, int bits, int mode, uint64_t seed,
                                 const int32_t* outlier_channels, int n_outlier, bool device,
                                 tq_quantizer** out) {
  if (!out) return TQ_EINVAL;
  *out = nullptr;
  tq_quantizer* q = new (std::nothrow) tq_quantizer;
  if (!q) return TQ_ENOMEM;
  std::memset(q, 0, sizeof(*q));
  tq_status st = build_host_tables(d, bits, mode, seed, outlier_channels, n_outlier, &q->host,
                                   &q->layout);
  if (st != TQ_OK) {
    delete q;
    return st;
  }
  q->d = d;
  q->bits = bits;
  q->mode = mode;
  q->seed = seed;
  q->device = -1;
  if (!device) {  // host-only: layouts and argument checks, no device tables
    *out = q;
    return TQ_OK;
  }

  DevTables* h = new (std::nothrow) DevTables;
  if (!h) {
    delete q;
    return TQ_ENOMEM;
  }
  std::memset(h, 0, sizeof(*h));
  const int nl0 = mode == TQ_MODE_MSE ? (1 << bits) : mode == TQ_MODE_PROD ? (1 << (bits - 1)) : (1 << (bits + 1));
  for (int k = 0; k < nl0; ++k) h->cent[0][k] = static_cast<float>(q->host.cent[0][k]);
  for (int k = 0; k + 1 < nl0; ++k) h->thr[0][k] = static_cast<float>(q->host.thr[0][k]);
  if (mode == TQ_MODE_GROUPED) {
    const int nl1 = 1 << bits;
    for (int k = 0; k < nl1; ++k) h->cent[1][k] = static_cast<float>(q->host.cent[1][k]);
    for (int k = 0; k + 1 < nl1; ++k) h->thr[1][k] = static_cast<float>(q->host.thr[1][k]);
  }
  for (int j = 0; j < kD; ++j) {
    if (q->host.signs[j] < 0) h->sign_bits[j >> 5] |= 1u << (j & 31);
    h->chan[j] = static_cast<uint8_t>(q->host.chan[j]);
  }
  if (mode == TQ_MODE_PROD) {
    for (int r = 0; r < kD; ++r)
      for (int c = 0; c < kD; ++c) {
        const uint16_t v = q->host.s_rot[r * kD + c];
        std::memcpy(&h->s_rot[r * kD + c], &v, 2);
        std::memcpy(&h->s_rot_t[c * kD + r], &v, 2);
      }
    for (int j = 0; j < kD; ++j)
      for (int kk = 0; kk < kD; ++kk) {
        const int col = (kk >> 1) + 64 * (kk & 1);
        const size_t off = static_cast<size_t>(j >> 3) * 1024 + (kk >> 3) * 64 + (j & 7) * 8 + (kk & 7);
        h->s_umma[off] = q->host.s_rot[j * kD + col];
      }
  }
  if (mode == TQ_MODE_GROUPED) gather_schedule(q->host.chan, h->gsched);
  for (int qq = 0; qq < kD / 2; ++qq)
    h->pair_mask[qq] = (q->host.signs[2 * qq] < 0 ? 1u << 15 : 0u) |
                       (q->host.signs[2 * qq + 1] < 0 ? 1u << 31 : 0u);
  if (cudaGetDevice(&q->device) != cudaSuccess) {
    delete h;
    delete q;
    return TQ_ECUDA;
  }
  if (cudaMalloc(&q->dev, sizeof(DevTables)) != cudaSuccess) {
    delete h;
    delete q;
    return TQ_ENOMEM;
  }
  st = cudaMemcpy(q->dev, h, sizeof(DevTables), cudaMemcpyHostToDevice) == cudaSuccess ? TQ_OK : TQ_ECUDA;
  delete h;
  if (st != TQ_OK) {
    cudaFree(q->dev);
    delete q;
    return st;
  }
  *out = q;
  return TQ_OK;
}

tq_status tq_build_codebook(int d, int bits, int mode, uint64_t seed,
                            const int32_t* outlier_channels, int n_outlier, tq_quantizer** out) {
  return build_quantizer(d, bits, mode, seed, outlier_channels, n_outlier, true, out);
}

tq_status tq_build_codebook_host(int d, int bits, int mode, uint64_t seed,
                                 const int32_t* outlier_channels, int n_outlier,
                                 tq_quantizer** out) {
  return build_quantizer(d, bits, mode, seed, outlier_channels, n_outlier, false, out);
}

void tq_free(tq_quantizer* q) {
  if (!q) return;
  if (q->dev) cudaFree(q->dev);
  delete q;
}

tq_status tq_key_layout(const tq_quantizer* q, tq_key_layout_t* out) {
  if (!q || !out) return TQ_EINVAL;
  *out = q->layout;
  return TQ_OK;
}

tq_status tq_quantize_keys(const tq_quantizer* q, const void* x, int dtype, int64_t n_rows,
                           int64_t ld, tq_key_planes out, void* stream) {
  if (!q) return TQ_EINVAL;
  tq_status st = check_rows(x, dtype, n_rows, ld);
  if (st != TQ_OK) return st;
  if (n_rows == 0) return TQ_OK;
  if ((st = check_key_planes(q, out)) != TQ_OK) return st;
  if (q->mode != TQ_MODE_GROUPED && (reinterpret_cast<uintptr_t>(out.norms) & 3u)) return TQ_EINVAL;
  if (!q->dev) return TQ_ECUDA;
  return launch_quantize_keys(q, x, dtype, n_rows, ld, out, RowMap{nullptr, 0, 0, 0},
                              static_cast<cudaStream_t>(stream));
}

tq_status tq_dequantize_keys(const tq_quantizer* q, tq_key_planes planes, int64_t n_rows,
                             void* out, int out_dtype, int64_t ld, void* stream) {
  if (!q) return TQ_EINVAL;
  tq_status st = check_rows(out, out_dtype, n_rows, ld);
  if (st != TQ_OK) return st;
  if (n_rows == 0) return TQ_OK;
  if ((st = check_key_planes(q, planes)) != TQ_OK) return st;
  if (!q->dev) return TQ_ECUDA;
  return launch_dequantize_keys(q, planes, n_rows, out, out_dtype, ld,
                                static_cast<cudaStream_t>(stream));
}

tq_status tq_quantize_values(const void* v, int dtype, int64_t n_rows, int64_t ld, int d, int bits,
                             int group, tq_value_planes out, void* stream) {
  if (d != kD) return TQ_EUNSUPPORTED;
  if (bits != 2 && bits != 4) return TQ_EUNSUPPORTED;
  if (group != 32) return TQ_EUNSUPPORTED;
  tq_status st = check_rows(v, dtype, n_rows, ld);
  if (st != TQ_OK) return st;
  if (n_rows == 0) return TQ_OK;
  if (!out.q || !out.params || (reinterpret_cast<uintptr_t>(out.params) & 3u) ||
      (reinterpret_cast<uintptr_t>(out.q) & 3u))
    return TQ_EINVAL;
  return launch_quantize_values(v, dtype, n_rows, ld, bits, out, RowMap{nullptr, 0, 0, 0},
                                static_cast<cudaStream_t>(stream));
}

// Argument checks of tq_append (nothing launched).
static tq_status check_append(const tq_quantizer* q, const tq_kv_cache* c, const void* k_new,
                              const void* v_new, int dtype, int n_tokens) {
  if (!q) return TQ_EINVAL;
  tq_status st = check_cache(q, c);
  if (st != TQ_OK) return st;
  if (n_tokens < 0) return TQ_EINVAL;
  if (n_tokens == 0) return TQ_OK;
  if (dtype != TQ_F32 && dtype != TQ_BF16) return TQ_EUNSUPPORTED;
  if (!k_new || !aligned16(k_new)) return TQ_EINVAL;
  if (c->value_bits != 0 && (!v_new || !aligned16(v_new))) return TQ_EINVAL;
  if (c->value_bits == 0 && v_new) return TQ_EINVAL;
  for (int b = 0; b < c->batch; ++b)
    if (static_cast<int64_t>(c->len_host[b]) + n_tokens > c->capacity) return TQ_ECAPACITY;
  return TQ_OK;
}

tq_status tq_append(const tq_quantizer* q, tq_kv_cache* c, const void* k_new, const void* v_new,
                    int dtype, int n_tokens, void* stream) {
  tq_status st = check_append(q, c, k_new, v_new, dtype, n_tokens);
  if (st != TQ_OK || n_tokens == 0) return st;
  if (!q->dev) return TQ_ECUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (append_fused_ok(q, c, n_tokens)) {
    if ((st = launch_append_fused(q, c, k_new, v_new, dtype, n_tokens, s)) != TQ_OK) return st;
    for (int b = 0; b < c->batch; ++b) c->len_host[b] += n_tokens;
    return TQ_OK;
  }
  const int64_t rows = static_cast<int64_t>(c->batch) * c->n_kv_heads * n_tokens;
  const RowMap map{c->len_dev, c->n_kv_heads, n_tokens, c->capacity};
  if ((st = launch_quantize_keys(q, k_new, dtype, rows, kD, c->keys, map, s)) != TQ_OK) return st;
  if (c->value_bits != 0) {
    if ((st = launch_quantize_values(v_new, dtype, rows, kD, c->value_bits, c->values, map, s)) != TQ_OK)
      return st;
  }
  if ((st = launch_advance_len(c->len_dev, c->batch, n_tokens, s)) != TQ_OK) return st;
  for (int b = 0; b < c->batch; ++b) c->len_host[b] += n_tokens;
  return TQ_OK;
}

tq_status tq_decode_workspace_bytes(const tq_kv_cache* c, int n_q_heads, size_t* bytes) {
  if (!c || !bytes || n_q_heads <= 0 || c->batch <= 0 || c->capacity <= 0) return TQ_EINVAL;
  *bytes = decode_workspace_bytes(c->batch, n_q_heads, c->capacity);
  return TQ_OK;
}

// Argument checks of every decode entry point (the workspace apart: check_workspace).
static tq_status check_decode_args(const tq_quantizer* q, const tq_kv_cache* c, const void* qv,
                                   int q_dtype, int n_q_heads, const int32_t* head_map,
                                   void* out, int out_dtype, float* scores, int64_t scores_ld) {
  if (!q) return TQ_EINVAL;
  tq_status st = check_cache(q, c);
  if (st != TQ_OK) return st;
  if (n_q_heads <= 0 || n_q_heads > 512) return TQ_EINVAL;
  if (q_dtype != TQ_F32 && q_dtype != TQ_BF16) return TQ_EUNSUPPORTED;
  if (!qv || !aligned16(qv)) return TQ_EINVAL;
  if (head_map) {
    for (int h = 0; h < n_q_heads; ++h)
      if (head_map[h] < 0 || head_map[h] >= c->n_kv_heads) return TQ_EINVAL;
  } else if (n_q_heads % c->n_kv_heads != 0) {
    return TQ_EINVAL;
  }
  if (c->value_bits != 0) {
    if (!out || !aligned16(out)) return TQ_EINVAL;
    if (out_dtype != TQ_F32 && out_dtype != TQ_BF16) return TQ_EUNSUPPORTED;
  } else if (out) {
    return TQ_EINVAL;
  }
  int max_len = 0;
  for (int b = 0; b < c->batch; ++b) max_len = c->len_host[b] > max_len ? c->len_host[b] : max_len;
  if (scores && scores_ld < max_len) return TQ_EINVAL;
  return TQ_OK;
}

static tq_status check_workspace(const tq_kv_cache* c, int n_q_heads, const void* workspace,
                                 size_t workspace_bytes) {
  if (!workspace || !aligned16(workspace)) return TQ_EINVAL;
  if (workspace_bytes < decode_workspace_bytes(c->batch, n_q_heads, c->capacity)) return TQ_EINVAL;
  return TQ_OK;
}

tq_status tq_decode_attention(const tq_quantizer* q, const tq_kv_cache* c, const void* qv,
                              int q_dtype, int n_q_heads, const int32_t* head_map, float sm_scale,
                              void* out, int out_dtype, float* scores, int64_t scores_ld,
                              void* workspace, size_t workspace_bytes, void* stream) {
  tq_status st = check_decode_args(q, c, qv, q_dtype, n_q_heads, head_map, out, out_dtype,
                                   scores, scores_ld);
  if (st != TQ_OK) return st;
  if ((st = check_workspace(c, n_q_heads, workspace, workspace_bytes)) != TQ_OK) return st;
  return launch_decode(q, c, qv, q_dtype, n_q_heads, head_map, sm_scale, out, out_dtype, scores,
                       scores_ld, nullptr, workspace, workspace_bytes, /*pdl=*/false,
                       static_cast<cudaStream_t>(stream));
}

tq_status tq_append_decode(const tq_quantizer* q, tq_kv_cache* c, const void* k_new,
                           const void* v_new, int kv_dtype, int n_tokens, const void* qv,
                           int q_dtype, int n_q_heads, const int32_t* head_map, float sm_scale,
                           void* out, int out_dtype, float* scores, int64_t scores_ld,
                           void* workspace, size_t workspace_bytes, void* stream) {
  tq_status st = check_append(q, c, k_new, v_new, kv_dtype, n_tokens);
  if (st != TQ_OK) return st;
  if ((st = check_decode_args(q, c, qv, q_dtype, n_q_heads, head_map, out, out_dtype, scores,
                              scores_ld)) != TQ_OK)
    return st;
  if (scores) {  // the scores cover the lengths after the append
    for (int b = 0; b < c->batch; ++b)
      if (static_cast<int64_t>(c->len_host[b]) + n_tokens > scores_ld) return TQ_EINVAL;
  }
  if ((st = check_workspace(c, n_q_heads, workspace, workspace_bytes)) != TQ_OK) return st;
  // the decode's head grouping is checked before the append, so that an error leaves the
  // cache as it was
  if ((st = check_decode_plan(q, c, n_q_heads, head_map, n_tokens)) != TQ_OK) return st;
  if (!q->dev) return TQ_ECUDA;
  if ((st = tq_append(q, c, k_new, v_new, kv_dtype, n_tokens, stream)) != TQ_OK) return st;
  // the kernel just launched is the library's append, ordered after the query's producer:
  // the decode may start its query-only prologue while the append runs
  return launch_decode(q, c, qv, q_dtype, n_q_heads, head_map, sm_scale, out, out_dtype, scores,
                       scores_ld, nullptr, workspace, workspace_bytes, /*pdl=*/true,
                       static_cast<cudaStream_t>(stream));
}

tq_status tq_decode_attention_partial(const tq_quantizer* q, const tq_kv_cache* c, const void* qv,
                                      int q_dtype, int n_q_heads, const int32_t* head_map,
                                      float sm_scale, float* part, void* workspace,
                                      size_t workspace_bytes, void* stream) {
  if (!q || !c) return TQ_EINVAL;
  if (c->value_bits == 0) return TQ_EINVAL;  // a partial carries o: the cache needs values
  if (!part || !aligned16(part)) return TQ_EINVAL;
  // every other check is tq_decode_attention's (with a stand-in output pointer)
  tq_status st = check_decode_args(q, c, qv, q_dtype, n_q_heads, head_map, part, TQ_F32,
                                   nullptr, 0);
  if (st != TQ_OK) return st;
  if ((st = check_workspace(c, n_q_heads, workspace, workspace_bytes)) != TQ_OK) return st;
  return launch_decode(q, c, qv, q_dtype, n_q_heads, head_map, sm_scale, nullptr, TQ_F32, nullptr,
                       0, part, workspace, workspace_bytes, /*pdl=*/false,
                       static_cast<cudaStream_t>(stream));
}

tq_status tq_set_decode_policy(int policy, int* previous) {
  return set_decode_policy(policy, previous);
}

tq_status tq_merge_partials(const float* parts, int n_parts, int batch, int n_q_heads, void* out,
                            int out_dtype, void* stream) {
  if (n_parts < 1 || n_parts > 65536 || batch <= 0 || n_q_heads <= 0 || n_q_heads > 512)
    return TQ_EINVAL;
  if (out_dtype != TQ_F32 && out_dtype != TQ_BF16) return TQ_EUNSUPPORTED;
  if (!parts || !aligned16(parts) || !out || !aligned16(out)) return TQ_EINVAL;
  return launch_merge_partials(parts, n_parts, static_cast<int64_t>(batch) * n_q_heads, out,
                               out_dtype, static_cast<cudaStream_t>(stream));
}

tq_status tq_decode_attention_noalloc(const tq_quantizer* q, const tq_kv_cache* c,
                                      const void* qv, int q_dtype, int n_q_heads,
                                      const int32_t* head_map, float sm_scale, void* out,
                                      int out_dtype, float* scores, int64_t scores_ld,
                                      void* stream) {
  tq_status st = check_decode_args(q, c, qv, q_dtype, n_q_heads, head_map, out, out_dtype,
                                   scores, scores_ld);
  if (st != TQ_OK) return st;
  if ((st = check_decode_plan(q, c, n_q_heads, head_map, 0)) != TQ_OK) return st;
  if (!q->dev) return TQ_ECUDA;
  return launch_decode_noalloc(q, c, qv, q_dtype, n_q_heads, head_map, sm_scale, out, out_dtype,
                               scores, scores_ld, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
