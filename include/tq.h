/*
 * tq.h -- C ABI of the B200 TurboQuant KV-cache library (libtq.so).
 *
 * TurboQuant compresses attention keys with a random rotation (Hadamard x random signs), a
 * Lloyd-Max Gaussian codebook per coordinate and, in "prod" mode, a 1-bit QJL sketch of the
 * residual; values use 2/4-bit asymmetric group quantization. Decode attention scores the
 * packed keys directly and sums the dequantized values.
 *
 * Sources (page title and section):
 *   tqlite README                      -- rotation.py "Hadamard x random signs", codebook.py
 *                                         Lloyd-Max Gaussian codebook, the "three quantization
 *                                         modes" table (mse, prod, grouped), design notes
 *                                         (per-row L2 normalisation, per-layer seeds).
 *   Implementing TurboQuant (part 5)   -- algorithm overview: residual, QJL sign(S @ r),
 *                                         estimator <q,k_hat> + sqrt(pi/2) (Sq)^T sign_bits.
 *   TurboQuant bit-packing article     -- sections 2-4: byte layouts of 2-bit, 4-bit (3-bit in
 *                                         4-bit fields) and sign planes, fp16 norms, 52 B/key;
 *                                         section 5: fused decode kernels read packed bytes,
 *                                         chunked append store.
 *   validate_paper.py                  -- TurboQuantMSE/Prod(dim, bits, seed), quantize,
 *                                         attention_score, CompressedKVStore(head_dim,
 *                                         num_kv_heads, key_bits, value_bits, group 32).
 *
 * Conventions for every entry point:
 *   - Pointers named *_dev are CUDA device memory owned by the caller; the library keeps no
 *     reference to them after the call returns. Host pointers are read during the call only.
 *   - Compute calls are asynchronous on `stream` (a cudaStream_t passed as void*, NULL = the
 *     legacy default stream). They allocate nothing.
 *   - Arguments are checked on the host before anything is launched; a bad argument returns
 *     TQ_EINVAL / TQ_EUNSUPPORTED / TQ_ECAPACITY and launches nothing. A launch failure
 *     returns TQ_ECUDA. Kernels never trap, assert or spin without a bound.
 *   - d = 128 on the GPU path. Rows are d contiguous elements; `ld` is the row stride in
 *     elements (>= d, and ld * element size a multiple of 16 bytes). Device pointers of row
 *     data and packed planes must be 16-byte aligned.
 */
#ifndef TQ_H
#define TQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define TQ_ABI_VERSION 1

typedef enum {
  TQ_OK = 0,
  TQ_EINVAL = -1,        /* bad argument (null pointer, size, alignment, mismatch) */
  TQ_EUNSUPPORTED = -2,  /* well-formed but not supported (d != 128 on GPU, bits, dtype) */
  TQ_ECAPACITY = -3,     /* cache would overflow: len + n_tokens > capacity */
  TQ_ENOMEM = -4,        /* host or device allocation failed (tq_build_codebook only) */
  TQ_ECUDA = -5,         /* a CUDA runtime call or kernel launch failed */
  TQ_ETIMEOUT = -6,      /* a bounded device wait gave up (tq_sync_status) */
  TQ_ETOOLARGE = -7      /* needs more scratch than tq_decode_attention_noalloc holds */
} tq_status;

enum { TQ_MODE_MSE = 0, TQ_MODE_PROD = 1, TQ_MODE_GROUPED = 2 };
enum { TQ_F32 = 0, TQ_BF16 = 1, TQ_F16 = 2 };

/* Opaque quantizer: codebook, rotation signs, QJL matrix, plus a small device copy. */
typedef struct tq_quantizer tq_quantizer;

/* Bytes per key of each packed plane (TurboQuant bit-packing article, section 4 ledger).
 *   mse  b : idx = d*w(b)/8, signs 0, norms 1 (||x||)                 18/34/66/66 B, b=1..4
 *   prod b : idx = d*w(b-1)/8, signs d/8, norms 2 (||x||, ||r||)     36/52/84 B,    b=2..4
 *   grouped b: idx = 32*w(b+1)/8 + 96*w(b)/8, signs 0, norms 2       24/44/68 B,    b=1..3
 * with storage width w(1)=1, w(2)=2, w(3)=w(4)=4 (3-bit codes in 4-bit fields). */
typedef struct {
  int32_t d, bits, mode;
  int32_t idx_bytes, sign_bytes, n_norms, bytes_per_key;
} tq_key_layout_t;

/* Packed key planes for n_rows keys, row-major, all device memory:
 *   idx   n_rows x idx_bytes   codebook indices; coordinate j of the rotated key sits at
 *                              bit (j*w) % 8 of byte (j*w)/8, lowest bits first
 *                              (2-bit: a | b<<2 | c<<4 | d<<6; 4-bit: a | b<<4).
 *                              grouped: [outlier-group codes | normal-group codes].
 *   signs n_rows x d/8         prod only (else NULL): QJL bit j = [(S r)_j >= 0], bit j%8 of
 *                              byte j/8 (weights 1,2,...,128).
 *   norms n_rows x n_norms     IEEE fp16 bit patterns: mse ||x||; prod ||x||, ||r||;
 *                              grouped ||x_outlier||, ||x_normal||. */
typedef struct {
  uint8_t* idx;
  uint8_t* signs;
  uint16_t* norms;
} tq_key_planes;

/* Packed value planes for n_rows value vectors (device memory):
 *   q      n_rows x d*bits/8        codes, packed like the key indices (2-bit or 4-bit)
 *   params n_rows x (d/group) x 2   fp16 bit patterns (min, scale) of each group */
typedef struct {
  uint8_t* q;
  uint16_t* params;
} tq_value_planes;

/* A preallocated packed KV cache (caller-owned device memory).
 * Row (b, h, t) of every plane is at ((b * n_kv_heads + h) * capacity + t).
 * capacity must be a multiple of 16. value_bits = 0 makes a key-only cache (values NULL).
 * len_dev[b] tokens are valid in sequence b; len_host mirrors it on the host and is the
 * copy the library checks capacity against and updates in tq_append. */
typedef struct {
  int32_t batch, n_kv_heads, capacity, d;
  int32_t value_bits, value_group;
  tq_key_planes keys;
  tq_value_planes values;
  int32_t* len_dev;
  int32_t* len_host;
} tq_kv_cache;

/* ------------------------------------------------------------------ set-up (host) */

/* Build a quantizer: Lloyd-Max codebook(s) of N(0,1) (tqlite codebook.py), the seeded
 * rotation signs (tqlite rotation.py) and, for prod, the seeded d x d Gaussian S_rot of the
 * QJL sketch; then copy them to the current CUDA device.
 *   d        128 (GPU); bits: mse 1..4, prod 2..4 (total, = (bits-1)-bit MSE + 1 QJL bit),
 *            grouped 1..3 (normal channels at bits, outlier channels at bits+1).
 *   seed     quantizer seed (one per layer, tqlite design notes); random numbers come from
 *            SplitMix64 streams of the seed (Steele, Lea & Flood 2014).
 *   outlier_channels / n_outlier: host array of 32 distinct channels in [0, d), grouped
 *            mode only (else NULL / 0).
 * On success *out owns a small device table until tq_free. Errors: TQ_EINVAL,
 * TQ_EUNSUPPORTED, TQ_ENOMEM, TQ_ECUDA (no device). */
tq_status tq_build_codebook(int d, int bits, int mode, uint64_t seed,
                            const int32_t* outlier_channels, int n_outlier,
                            tq_quantizer** out);

/* The same quantizer without a device copy of its tables, built on the host alone (no GPU
 * needed): for plane sizes (tq_key_layout) and for checking arguments before device memory
 * exists. Every device entry point given it runs its argument checks (and returns their
 * errors) and then returns TQ_ECUDA without launching anything or changing the cache.
 * Free it with tq_free. Errors as tq_build_codebook (no TQ_ECUDA). */
tq_status tq_build_codebook_host(int d, int bits, int mode, uint64_t seed,
                                 const int32_t* outlier_channels, int n_outlier,
                                 tq_quantizer** out);

void tq_free(tq_quantizer* q);

/* Plane sizes of a quantizer's keys (host only). */
tq_status tq_key_layout(const tq_quantizer* q, tq_key_layout_t* out);

/* The host tables behind a quantizer, for inspection (host only, no device needed):
 *   centroids[2*16], thresholds[2*16]  N(0,1)-scale Lloyd-Max levels and cell edges,
 *                       ascending; row 0 = main (grouped: outlier group), row 1 = grouped
 *                       normal group; unused entries are 0.
 *   signs[128]          rotation signs (+1/-1); grouped: 32 outlier-group signs followed by
 *                       96 normal-group signs.
 *   channels[128]       grouped: the 32 outlier channels ascending then the 96 others
 *                       ascending; otherwise 0..d-1.
 *   s_rot_fp16[d*d]     prod: S_rot row-major as fp16 bits; may be NULL. */
tq_status tq_host_tables(int d, int bits, int mode, uint64_t seed,
                         const int32_t* outlier_channels, int n_outlier,
                         double* centroids, double* thresholds, int8_t* signs,
                         int32_t* channels, uint16_t* s_rot_fp16);

/* ------------------------------------------------------------------ hot path (device) */

/* Quantize n_rows keys x_dev (n_rows x ld, dtype TQ_F32 or TQ_BF16) into `out`
 * (tqlite mse.py / prod.py / grouped.py; bit-packing article sections 2-4).
 * Per row: n = ||x||; u = Pi x / n; idx_j = #{k : u_j > t_k}; prod adds r = x - x_mse,
 * ||r|| and the QJL signs [(S r)_j >= 0] with S = S_rot Pi. n_rows = 0 is a no-op. */
tq_status tq_quantize_keys(const tq_quantizer* q, const void* x_dev, int dtype,
                           int64_t n_rows, int64_t ld, tq_key_planes out, void* stream);

/* Dequantize n_rows packed keys (`planes`, the layout tq_quantize_keys writes) into out_dev
 * (n_rows x ld, TQ_F32 or TQ_BF16, same row rules as tq_quantize_keys' input), in the
 * original coordinates (validate_paper.py dequantize; tqlite prod.py):
 *   mse:     x_hat = ||x|| Pi^T c[idx]
 *   prod:    x_hat = ||x|| Pi^T c[idx] + ||r|| sqrt(pi/2)/d S^T (2 sigma - 1)   (S = S_rot Pi),
 *            so that <q, x_hat> equals the decode estimator s(q)
 *   grouped: each group's mse reconstruction on its own channels.
 * n_rows = 0 is a no-op. Not part of the decode hot path (quality checks, debugging). */
tq_status tq_dequantize_keys(const tq_quantizer* q, tq_key_planes planes, int64_t n_rows,
                             void* out_dev, int out_dtype, int64_t ld, void* stream);

/* Quantize n_rows value vectors v_dev (n_rows x ld, TQ_F32 or TQ_BF16; d = 128) into
 * `out`: per group of `group` (= 32) channels, mn = min, scale = (max - mn)/(2^bits - 1),
 * stored as fp16; code = clamp(rint((v - mn16)/s16), 0, 2^bits - 1), 0 if s16 = 0; the
 * code decision uses fp32 IEEE subtract and divide (bit-packing article sections 2-3).
 * bits = 2 or 4. */
tq_status tq_quantize_values(const void* v_dev, int dtype, int64_t n_rows, int64_t ld,
                             int d, int bits, int group, tq_value_planes out, void* stream);

/* Append n_tokens new keys (and values) per (batch, KV head) to the cache: token t of
 * (b, h) is quantized and written at position len[b] + t, then len[b] += n_tokens on the
 * device and in len_host (bit-packing article section 5, store.py append).
 * k_new_dev / v_new_dev: batch x n_kv_heads x n_tokens x d, dtype TQ_F32 or TQ_BF16,
 * contiguous; v_new_dev must be NULL for a key-only cache. Returns TQ_ECAPACITY (nothing
 * launched) if any len_host[b] + n_tokens > capacity. */
tq_status tq_append(const tq_quantizer* q, tq_kv_cache* cache, const void* k_new_dev,
                    const void* v_new_dev, int dtype, int n_tokens, void* stream);

/* One decode step: tq_append of this step's tokens followed by tq_decode_attention, both on
 * `stream`. The decode is launched with programmatic dependent launch right behind the
 * library's own append kernel, so that its query-only prologue (query rotation, S q, lookup
 * tables) overlaps the append; it reads the lengths and the cache only once the append has
 * completed. The query must be ready when this call's first kernel starts (written by work
 * ordered before the call on `stream`), which stream order already guarantees. Arguments are
 * those of the two calls (k_new_dev / v_new_dev / kv_dtype / n_tokens for the append; the
 * rest for the decode) and are all checked before anything is launched, including the
 * decode's head grouping for the lengths after the append: on any error nothing is launched
 * and the cache is unchanged; the first error is returned. */
tq_status tq_append_decode(const tq_quantizer* q, tq_kv_cache* cache, const void* k_new_dev,
                           const void* v_new_dev, int kv_dtype, int n_tokens,
                           const void* q_dev, int q_dtype, int n_q_heads,
                           const int32_t* head_map, float sm_scale, void* out_dev, int out_dtype,
                           float* scores_dev, int64_t scores_ld,
                           void* workspace_dev, size_t workspace_bytes, void* stream);

/* Workspace bytes tq_decode_attention needs for this cache and query-head count. The
 * workspace must be zero-filled before its first use; every call leaves it reusable. */
tq_status tq_decode_workspace_bytes(const tq_kv_cache* cache, int n_q_heads, size_t* bytes);

/* Fused decode attention over a packed cache of any key mode, one query token per sequence.
 * For query head h of sequence b with KV head kv = head_map[h], and every i < len[b]:
 *   prod:    s_i = ||x_i|| <Pi q, c[idx_i]> + ||r_i|| sqrt(pi/2)/d <S q, 2 sigma_i - 1>
 *   mse:     s_i = ||x_i|| <Pi q, c[idx_i]>
 *   grouped: s_i = sum over the two channel groups g of ||x_i,g|| <Pi_g q_g, c_g[idx_i,g]>
 *   out = softmax(sm_scale * s) . v_hat,   v_hat = mn16 + code * s16.
 * The kernel is an ordinary launch on `stream`: every earlier work on the stream (the query's
 * producer included) has completed when it starts.
 * q_dev: batch x n_q_heads x d (TQ_F32 or TQ_BF16). head_map: host int32[n_q_heads] with
 * values in [0, n_kv_heads), NULL = h / (n_q_heads / n_kv_heads). sm_scale <= 0 means
 * 1/sqrt(d). out_dev: batch x n_q_heads x d in out_dtype (TQ_F32 or TQ_BF16), may be NULL
 * only for a key-only cache. scores_dev (nullable): fp32 batch x n_q_heads x scores_ld raw
 * estimates s_i for i < len[b] (scores_ld >= max len). A sequence with len 0 yields zeros. */
tq_status tq_decode_attention(const tq_quantizer* q, const tq_kv_cache* cache,
                              const void* q_dev, int q_dtype, int n_q_heads,
                              const int32_t* head_map, float sm_scale,
                              void* out_dev, int out_dtype,
                              float* scores_dev, int64_t scores_ld,
                              void* workspace_dev, size_t workspace_bytes, void* stream);

/* tq_decode_attention without a workspace argument, for callers that cannot allocate
 * device memory: for example a plain C host with no device allocator of its own, or a
 * serving loop that must not call cudaMalloc on its hot path (cudaMalloc can synchronize
 * the device and its latency is unbounded). The paper has no counterpart; this is a
 * convenience of the library.
 *
 * The scratch the decode kernel needs (per-split partial results and split counters)
 * lives in one file-scope device array of TQ_NOALLOC_SCRATCH_BYTES (16 MiB) that every
 * GPU loading the library holds until the process exits. Problems whose scratch
 * (tq_decode_workspace_bytes) exceeds it return TQ_ETOOLARGE and launch nothing.
 * The first call on a device looks up the array's device address (once per device, with
 * that device current); make that first call before any stream capture. Each call clears
 * the split counters it uses (an async memset on `stream`) and allocates nothing. All
 * calls share the one array: calls whose kernels overlap on the GPU (other streams, other
 * host threads) race on it and must be serialised by the caller. Arguments and results are
 * otherwise exactly those of tq_decode_attention. */
#define TQ_NOALLOC_SCRATCH_BYTES (16u << 20)
tq_status tq_decode_attention_noalloc(const tq_quantizer* q, const tq_kv_cache* cache,
                                      const void* q_dev, int q_dtype, int n_q_heads,
                                      const int32_t* head_map, float sm_scale,
                                      void* out_dev, int out_dtype,
                                      float* scores_dev, int64_t scores_ld, void* stream);

/* Shape of the fused decode's thread blocks (process-wide; a tuning and testing knob, the
 * results do not depend on it beyond fp32 rounding order). A block scores and sums the
 * tokens of one KV head for a group of its query heads. TQ_DECODE_AUTO (the default): groups
 * of up to 8 query heads (two 4-head lookup-table sets, 8 warps) when a KV head has more
 * than 4, the two-set tables fit the shared memory and the decode holds at least 4 x 256
 * (token, KV head) units per SM; else groups of up to 4 (one table set, 16 warps). Grouped
 * keys always use one set. TQ_DECODE_TWO_SETS drops the size condition; TQ_DECODE_ONE_SET
 * forces groups of up to 4. Writes the previous policy to `previous` (nullable); TQ_EINVAL
 * for another value (nothing changed). */
#define TQ_DECODE_AUTO 0
#define TQ_DECODE_ONE_SET 1
#define TQ_DECODE_TWO_SETS 2
tq_status tq_set_decode_policy(int policy, int* previous);

/* ---- context-parallel decode (a cache's context split into slices, e.g. one per GPU) ----
 * Softmax attention over the union of the slices equals the LSE merge of per-slice partial
 * results (the merge the fused decode kernel already runs between its own context splits):
 *   step 1, per slice:  tq_decode_attention_partial -> (m, l, o) per (sequence, query head)
 *   exchange:           gather every slice's records (an all-gather across GPUs)
 *   step 2:             tq_merge_partials -> out = sum 2^(m_r - M) o_r / sum 2^(m_r - M) l_r
 * A record is TQ_PART_FLOATS fp32 values: m (the largest logit, base 2: sm_scale log2(e) s),
 * l = sum_i 2^(x_i - m), two zeros, and the unnormalised o = sum_i 2^(x_i - m) v_hat_i [d].
 * An empty slice (len[b] = 0) gives m = -inf, l = 0, o = 0. */
#define TQ_PART_FLOATS 132

/* Step 1: as tq_decode_attention (same arguments, checks and workspace) on a cache with
 * values, writing the records to part_dev (fp32 batch x n_q_heads x TQ_PART_FLOATS,
 * 16-byte aligned) instead of normalised outputs. */
tq_status tq_decode_attention_partial(const tq_quantizer* q, const tq_kv_cache* cache,
                                      const void* q_dev, int q_dtype, int n_q_heads,
                                      const int32_t* head_map, float sm_scale, float* part_dev,
                                      void* workspace_dev, size_t workspace_bytes, void* stream);

/* Step 2: merge n_parts (1 .. 65536) slices' records, parts_dev = fp32 n_parts x batch x
 * n_q_heads x TQ_PART_FLOATS (16-byte aligned; slices may come in any order), into out_dev
 * (batch x n_q_heads x d, TQ_F32 or TQ_BF16, 16-byte aligned). All slices must have used the
 * same sm_scale. */
tq_status tq_merge_partials(const float* parts_dev, int n_parts, int batch, int n_q_heads,
                            void* out_dev, int out_dtype, void* stream);

/* Wait for `stream` (cudaStream_t as void*, NULL = legacy default stream) and report whether
 * any library kernel since the previous call gave up one of its bounded device waits (an
 * mbarrier wait on a bulk copy or a tensor-core product, limit 2 s): TQ_ETIMEOUT if so (the
 * flag is then cleared, and the outputs of that kernel are incomplete), TQ_ECUDA if the
 * stream reports a CUDA error, else TQ_OK. The flag is per process and device, shared by
 * all streams. */
tq_status tq_sync_status(void* stream);

/* Diagnostic of the error path above: launches on `stream` a one-thread kernel that waits on
 * an mbarrier phase nothing completes and gives up after `limit_us` microseconds
 * (1 .. 2000000; else TQ_EINVAL, nothing launched), recording the timeout in the device flag
 * so that the next tq_sync_status returns TQ_ETIMEOUT. No device fault is involved. */
tq_status tq_selftest_bounded_wait(uint32_t limit_us, void* stream);

const char* tq_status_string(tq_status s);
int tq_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* TQ_H */
