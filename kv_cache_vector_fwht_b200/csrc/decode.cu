// Fused decode attention, host side: head groups, block shape and context splits of a launch,
// the LSE merge of context-parallel partial records, and the no-workspace entry point.
// The kernel itself is in decode_kernel.cuh (instantiated per key kind in decode_*.cu).
#include <algorithm>
#include <atomic>
#include <cmath>
#include <mutex>

#include "decode_kernel.cuh"

namespace tq {
namespace dec {

std::atomic<int> g_decode_policy{TQ_DECODE_AUTO};

bool two_sets_ok(int kind, int mb, int vb) {
  switch (kind * 64 + mb * 8 + vb) {
#define TQ_TWO(KIND, MB, VB) \
  case KIND * 64 + MB * 8 + VB: return two_sets_fit<MB, VB, KIND>();
    TQ_TWO(kProd, 1, 0) TQ_TWO(kProd, 1, 2) TQ_TWO(kProd, 1, 4)
    TQ_TWO(kProd, 2, 0) TQ_TWO(kProd, 2, 2) TQ_TWO(kProd, 2, 4)
    TQ_TWO(kProd, 3, 0) TQ_TWO(kProd, 3, 2) TQ_TWO(kProd, 3, 4)
    TQ_TWO(kMse, 1, 0) TQ_TWO(kMse, 1, 2) TQ_TWO(kMse, 1, 4)
    TQ_TWO(kMse, 2, 0) TQ_TWO(kMse, 2, 2) TQ_TWO(kMse, 2, 4)
    TQ_TWO(kMse, 3, 0) TQ_TWO(kMse, 3, 2) TQ_TWO(kMse, 3, 4)
    TQ_TWO(kMse, 4, 0) TQ_TWO(kMse, 4, 2) TQ_TWO(kMse, 4, 4)
#undef TQ_TWO
    default: return false;
  }
}

namespace {

int max_splits_for(int capacity) {
  const int s = (capacity + 255) / 256;
  return s < 1 ? 1 : (s > 256 ? 256 : s);
}

// LSE merge of context-split partial records (m, l, o) of n_parts slices: per row (sequence,
// query head) M = max m_r, out = sum 2^(m_r - M) o_r / sum 2^(m_r - M) l_r (zeros when every
// slice is empty). One warp per row, lane l owns channels 4l .. 4l + 3.
__global__ void __launch_bounds__(128) k_merge_partials(const float* __restrict__ parts, int n_parts,
                                                        int64_t rows, void* out, int out_f32) {
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  float M = -INFINITY;
  for (int r = 0; r < n_parts; ++r) M = fmaxf(M, __ldg(parts + (r * rows + row) * kPartStride));
  float L = 0.f;
  float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
  if (M != -INFINITY) {
    for (int r = 0; r < n_parts; ++r) {
      const float* rec = parts + (r * rows + row) * kPartStride;
      const float mr = __ldg(rec);
      if (mr == -INFINITY) continue;
      const float f = exp2f(mr - M);
      L = fmaf(f, __ldg(rec + 1), L);
      const float4 v = __ldg(reinterpret_cast<const float4*>(rec + 4) + lane);
      O.x = fmaf(f, v.x, O.x); O.y = fmaf(f, v.y, O.y);
      O.z = fmaf(f, v.z, O.z); O.w = fmaf(f, v.w, O.w);
    }
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  const int64_t orow = row * kD + 4 * lane;
  if (out_f32) {
    *reinterpret_cast<float4*>(static_cast<float*>(out) + orow) =
        make_float4(O.x * inv, O.y * inv, O.z * inv, O.w * inv);
  } else {
    __nv_bfloat162 lo = __floats2bfloat162_rn(O.x * inv, O.y * inv);
    __nv_bfloat162 hi = __floats2bfloat162_rn(O.z * inv, O.w * inv);
    uint2 pk;
    pk.x = *reinterpret_cast<uint32_t*>(&lo);
    pk.y = *reinterpret_cast<uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(static_cast<uint16_t*>(out) + orow) = pk;
  }
}

// The launch of one decode: argument block, grid and instantiation.
struct Plan {
  DecodeArgs a;
  dim3 grid;
  int kind, mb, vb, max_heads, n_groups;
  bool two;
};

// Head groups, block shape and context splits for the cache's host lengths plus `len_add`
// tokens (an append launched just before). TQ_EUNSUPPORTED when the groups exceed one
// launch; nothing is launched here.
tq_status plan_decode(const tq_quantizer* q, const tq_kv_cache* c, int n_q_heads,
                      const int32_t* head_map, int len_add, Plan* p) {
  DecodeArgs& a = p->a;
  p->kind = q->mode == TQ_MODE_PROD ? kProd : (q->mode == TQ_MODE_GROUPED ? kGrp : kMse);
  p->mb = p->kind == kProd ? q->bits - 1 : q->bits;
  p->vb = c->value_bits;

  int max_len = 0;
  for (int b = 0; b < c->batch; ++b) max_len = std::max(max_len, c->len_host[b] + len_add);
  int dev = 0;
  cudaGetDevice(&dev);
  const int sms = std::max(1, sm_count(dev) - 4);

  // query heads of each KV head (the default map: n_q_heads / n_kv_heads consecutive heads)
  const int per_default = head_map ? 0 : n_q_heads / c->n_kv_heads;
  int per_kv_max = per_default;
  if (head_map) {
    // heads mapped to each KV head that has any (head_map values are checked on entry)
    int seen_kv[kMaxQHeads], seen_n[kMaxQHeads], n_seen = 0;
    for (int h = 0; h < n_q_heads; ++h) {
      int i = 0;
      while (i < n_seen && seen_kv[i] != head_map[h]) ++i;
      if (i == n_seen) { seen_kv[n_seen] = head_map[h]; seen_n[n_seen++] = 0; }
      per_kv_max = std::max(per_kv_max, ++seen_n[i]);
    }
  }
  // Blocks of up to 8 query heads (two table sets) when some KV head has more than 4, the
  // two-set layout fits, and the decode is large enough to amortise the two-set block's
  // longer fixed path (twice the tables to build, more heads per chunk): at least 4 chunk
  // rounds of (token, KV head) units per SM. Measured: 1.05 M units (batch 8 x 4 KV heads x
  // 32768, or 1 x 8 x 131072) run 15-20 % faster with two sets; 65536 units (1 x 2 x 32768)
  // run 15 % slower. tq_set_decode_policy can force either shape.
  const int policy = g_decode_policy.load(std::memory_order_relaxed);
  const long long units = static_cast<long long>(c->batch) * c->n_kv_heads * max_len;
  p->two = per_kv_max > kSetHeads && two_sets_ok(p->kind, p->mb, p->vb) &&
           policy != TQ_DECODE_ONE_SET &&
           (policy == TQ_DECODE_TWO_SETS || units >= 4ll * Shape<2>::chunk_stride * sms);
  const int cap = p->two ? kMaxSlots : kSetHeads;

  // head groups: the query heads of each KV head, in balanced groups of at most `cap`
  int n_groups = 0, max_heads = 0, n_listed = 0;
  int heads[kMaxQHeads];
  for (int kv = 0; kv < c->n_kv_heads && n_listed < n_q_heads; ++kv) {
    int n = 0;
    if (head_map) {
      for (int h = 0; h < n_q_heads; ++h)
        if (head_map[h] == kv) heads[n++] = h;
    } else {
      for (int h = kv * per_default; h < (kv + 1) * per_default; ++h) heads[n++] = h;
    }
    if (n == 0) continue;
    const int ng = (n + cap - 1) / cap;
    int pos = 0;
    for (int g = 0; g < ng; ++g) {
      const int cnt = (n - pos) / (ng - g);
      if (n_groups >= kMaxGroups) return TQ_EUNSUPPORTED;
      a.group[n_groups] = group_word(kv, n_listed, cnt);
      for (int i = 0; i < cnt; ++i) a.heads[n_listed++] = static_cast<int16_t>(heads[pos + i]);
      max_heads = std::max(max_heads, cnt);
      pos += cnt;
      ++n_groups;
    }
  }
  p->max_heads = max_heads;
  p->n_groups = n_groups;

  // split count: one block per SM; minimise waves x (tokens per split + per-block set-up) +
  // the final combine (its loads grow with the number of splits). A few SMs are left out of
  // the first wave so that an append kernel still resident on them does not hold back a
  // block of this grid when it starts early (programmatic dependent launch).
  const int pairs = c->batch * std::max(1, n_groups);
  const int cap_splits = max_splits_for(c->capacity);
  const int chunk = p->two ? Shape<2>::chunk_stride : Shape<1>::chunk_stride;
  int best = 1;
  double best_cost = 1e300;
  const int max_try = std::max(1, std::min(cap_splits, (max_len + 255) / 256));
  for (int s = 1; s <= max_try; ++s) {
    const int tps = ((max_len + s - 1) / s + 31) & ~31;
    if ((max_len + tps - 1) / tps != s) continue;
    const double waves = std::ceil(static_cast<double>(pairs) * s / sms);
    const double cost = waves * (tps + chunk) + (s > 1 ? 8.0 * s : 0.0);
    if (cost < best_cost - 1e-9) { best_cost = cost; best = s; }
  }
  a.n_splits = best;
  a.max_len = max_len;
  a.tokens_per_split = std::max(32, ((max_len + best - 1) / best + 31) & ~31);
  p->grid = dim3(a.n_splits, std::max(1, n_groups), c->batch);
  return TQ_OK;
}

}  // namespace
}  // namespace dec

using namespace dec;

tq_status launch_merge_partials(const float* parts, int n_parts, int64_t rows, void* out,
                                int out_dtype, cudaStream_t st) {
  if (rows == 0) return TQ_OK;
  const int64_t blocks = (rows + 3) / 4;
  k_merge_partials<<<static_cast<unsigned>(blocks), 128, 0, st>>>(parts, n_parts, rows, out,
                                                                 out_dtype == TQ_F32);
  return cudaGetLastError() == cudaSuccess ? TQ_OK : TQ_ECUDA;
}

size_t decode_workspace_bytes(int batch, int n_q_heads, int capacity) {
  const size_t parts = static_cast<size_t>(batch) * n_q_heads * max_splits_for(capacity) *
                       kPartStride * sizeof(float);
  const size_t ctrs = static_cast<size_t>(batch) * n_q_heads * sizeof(int);
  return ((parts + 255) / 256) * 256 + ((ctrs + 255) / 256) * 256;
}

tq_status check_decode_plan(const tq_quantizer* q, const tq_kv_cache* c, int n_q_heads,
                            const int32_t* head_map, int len_add) {
  static thread_local Plan p;
  return plan_decode(q, c, n_q_heads, head_map, len_add, &p);
}

tq_status launch_decode(const tq_quantizer* q, const tq_kv_cache* c, const void* qv, int q_dtype,
                        int n_q_heads, const int32_t* head_map, float sm_scale, void* out,
                        int out_dtype, float* scores, int64_t scores_ld, float* part_out,
                        void* workspace, size_t workspace_bytes, bool pdl, cudaStream_t st) {
  static thread_local Plan p;
  tq_status s = plan_decode(q, c, n_q_heads, head_map, 0, &p);
  if (s != TQ_OK) return s;
  if (!q->dev) return TQ_ECUDA;  // a host-only quantizer: checks done, nothing to launch
  if (p.n_groups == 0) return TQ_OK;
  DecodeArgs& a = p.a;
  if (a.max_len == 0 && out == nullptr && part_out == nullptr) return TQ_OK;
  a.part_out = part_out;
  a.k_idx = c->keys.idx;
  a.k_sgn = c->keys.signs;
  a.k_nrm = c->keys.norms;
  a.v_q = c->values.q;
  a.v_par = c->values.params;
  a.len = c->len_dev;
  a.q = qv;
  a.out = out;
  a.scores = scores;
  a.scores_ld = scores_ld;
  a.tab = q->dev;
  a.err = device_error_word();
  a.n_kv_heads = c->n_kv_heads;
  a.capacity = c->capacity;
  a.n_q_heads = n_q_heads;
  a.q_f32 = q_dtype == TQ_F32;
  a.out_f32 = out_dtype == TQ_F32;
  const float scale = sm_scale > 0.f ? sm_scale : 1.f / std::sqrt(static_cast<float>(kD));
  a.scale_log2 = scale * 1.4426950408889634074f;
  a.inv_scale_log2 = 1.f / a.scale_log2;
  if (decode_workspace_bytes(c->batch, n_q_heads, c->capacity) > workspace_bytes) return TQ_EINVAL;
  const size_t parts = static_cast<size_t>(c->batch) * n_q_heads * max_splits_for(c->capacity) *
                       kPartStride * sizeof(float);
  a.part = static_cast<float*>(workspace);
  a.counters = reinterpret_cast<int*>(static_cast<uint8_t*>(workspace) + ((parts + 255) / 256) * 256);
  switch (p.kind) {
    case kProd: return launch_kind_prod(a, p.mb, p.vb, p.grid, p.max_heads, p.two, pdl, st);
    case kMse: return launch_kind_mse(a, p.mb, p.vb, p.grid, p.max_heads, p.two, pdl, st);
    case kGrp: return launch_kind_grp(a, p.mb, p.vb, p.grid, p.max_heads, p.two, pdl, st);
    default: return TQ_EUNSUPPORTED;
  }
}

// ---------------------------------------------------------------------------------------
// Decode without a caller workspace: the partials and split counters live in this file-scope
// device array (TQ_NOALLOC_SCRATCH_BYTES, held by every GPU that loads the library until the
// process exits). Host code cannot use the array's name as a device address; its address
// is looked up once per device with cudaGetSymbolAddress, with that device current.
// ---------------------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_noalloc_scratch[TQ_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_addr[kMaxDevices] = {};
}  // namespace

tq_status launch_decode_noalloc(const tq_quantizer* q, const tq_kv_cache* c, const void* qv,
                                int q_dtype, int n_q_heads, const int32_t* head_map,
                                float sm_scale, void* out, int out_dtype, float* scores,
                                int64_t scores_ld, cudaStream_t st) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TQ_ECUDA;
  void* base = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (g_scratch_addr[dev] == nullptr) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
        return TQ_ECUDA;
      g_scratch_addr[dev] = p;
    }
    base = g_scratch_addr[dev];
  }
  const size_t need = decode_workspace_bytes(c->batch, n_q_heads, c->capacity);
  if (need > TQ_NOALLOC_SCRATCH_BYTES) return TQ_ETOOLARGE;
  // the split counters must start at zero; earlier calls leave their last contents here
  const size_t parts = static_cast<size_t>(c->batch) * n_q_heads * max_splits_for(c->capacity) *
                       kPartStride * sizeof(float);
  const size_t ctr_off = ((parts + 255) / 256) * 256;
  const size_t ctr_bytes = static_cast<size_t>(c->batch) * n_q_heads * sizeof(int);
  if (cudaMemsetAsync(static_cast<unsigned char*>(base) + ctr_off, 0, ctr_bytes, st) != cudaSuccess)
    return TQ_ECUDA;
  return launch_decode(q, c, qv, q_dtype, n_q_heads, head_map, sm_scale, out, out_dtype, scores,
                       scores_ld, nullptr, base, need, /*pdl=*/false, st);
}

tq_status set_decode_policy(int policy, int* previous) {
  if (policy != TQ_DECODE_AUTO && policy != TQ_DECODE_ONE_SET && policy != TQ_DECODE_TWO_SETS)
    return TQ_EINVAL;
  const int old = g_decode_policy.exchange(policy);
  if (previous) *previous = old;
  return TQ_OK;
}

}  // namespace tq
