// Internal declarations of libtq: the device copy of a quantizer's tables, the host
// quantizer object and the kernel launchers. Not part of the public ABI (include/tq.h).
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "../../include/tq.h"

namespace tq {

constexpr int kD = 128;          // head dimension of the GPU path
constexpr int kMaxLevels = 16;   // 4-bit codebook

// Tables a kernel needs, in one device allocation per quantizer.
// Row 0 of thr/cent is the full-width quantizer (grouped: the outlier group), row 1 the
// grouped normal group. Thresholds and centroids are N(0,1)-scale: the kernels compare the
// unnormalised Hadamard transform y = H (s . x) of a d_g-channel group against
// t_k * ||x_g|| * sqrt(32 / d_g) (sqrt factor only for the 96-channel group), which is
// the decision u_j = (Pi x)_j / ||x|| > t_k / sqrt(d_g).
struct DevTables {
  float thr[2][kMaxLevels];
  float cent[2][kMaxLevels];
  uint32_t sign_bits[4];   // bit j set <=> rotation sign s_j = -1 (grouped: 32 outlier, 96 normal)
  uint8_t chan[kD];        // grouped: outlier channels ascending, then normal channels ascending
  __half s_rot[kD * kD];   // prod: S_rot row-major (fp16-exact Gaussian)
  __half s_rot_t[kD * kD]; // prod: S_rot transposed (column j of S_rot contiguous)
  // prod: S_rot as the tensor-core B operand image (fp16 bits): K order permuted so that
  // k' = 2p holds column p and k' = 2p + 1 column p + 64, laid out in the canonical K-major
  // no-swizzle form (element (j, k') at byte (j/8)*2048 + (k'/8)*128 + (j%8)*16 + (k'%8)*2).
  alignas(16) uint16_t s_umma[kD * kD];
  // rotation signs of bf16 element pairs: word q has bit 15 set if s_{2q} = -1, bit 31 if
  // s_{2q+1} = -1 (an XOR flips both elements of a packed pair).
  alignas(16) uint32_t pair_mask[kD / 2];
  // grouped: store order of the per-warp gather into chain order. Lane l holds natural
  // channels 4l .. 4l + 3; in store round k it writes channel 4l + gsched[l][k], chosen so that
  // the 32 lanes of a round write 32 different shared-memory banks.
  uint8_t gsched[32][4];
};

struct HostTables {
  double cent[2][kMaxLevels];
  double thr[2][kMaxLevels];
  int8_t signs[kD];
  int32_t chan[kD];
  uint16_t s_rot[kD * kD];  // fp16 bits
};

// Host set-up (tq_host.cpp).
tq_status build_host_tables(int d, int bits, int mode, uint64_t seed, const int32_t* outliers,
                            int n_outlier, HostTables* t, tq_key_layout_t* layout);
uint16_t float_to_half_bits_rn(double x);

}  // namespace tq

struct tq_quantizer {
  int d, bits, mode;
  uint64_t seed;
  tq_key_layout_t layout;
  tq::HostTables host;
  tq::DevTables* dev;   // device copy
  int device;           // CUDA device the copy lives on
};

namespace tq {

// ---------------------------------------------------------------- kernel launchers

// Where quantized rows are written. Contiguous: output row = input row. Cache: input row r
// = ((b * n_kv_heads + h) * n_tokens + t) goes to cache row (b * n_kv_heads + h) * capacity
// + len[b] + t, with len read on the device.
struct RowMap {
  const int32_t* len;   // nullptr => contiguous
  int32_t n_kv_heads, n_tokens, capacity;
};

tq_status launch_quantize_keys(const tq_quantizer* q, const void* x, int dtype, int64_t n_rows,
                               int64_t ld, tq_key_planes out, RowMap map, cudaStream_t st);
tq_status launch_quantize_values(const void* v, int dtype, int64_t n_rows, int64_t ld, int bits,
                                 tq_value_planes out, RowMap map, cudaStream_t st);
tq_status launch_advance_len(int32_t* len, int batch, int n, cudaStream_t st);
// packed key planes back to vectors in the original coordinates
tq_status launch_dequantize_keys(const tq_quantizer* q, tq_key_planes planes, int64_t n_rows,
                                 void* out, int out_dtype, int64_t ld, cudaStream_t st);
// prod-mode bf16 keys with the QJL projection on tcgen05 tensor cores
bool keys_tc_ok(const tq_quantizer* q, int dtype);
tq_status launch_keys_tc(const tq_quantizer* q, const void* x, int64_t n_rows, int64_t ld,
                         tq_key_planes out, RowMap map, cudaStream_t st);
// Device address of the error word that kernels set when a bounded wait runs out (the current
// device; nullptr if it cannot be looked up).
int* device_error_word();
// Synchronise `st`; TQ_ETIMEOUT (and clear the flag) if a kernel gave up a bounded wait.
tq_status take_device_error(cudaStream_t st);
// A one-thread kernel whose bounded mbarrier wait runs out (sets the error flag).
tq_status launch_selftest_wait(uint32_t limit_us, cudaStream_t st);

// Fused append of a few tokens (mse / prod keys + values + lengths in one launch).
constexpr int kMaxAppendBatch = 64;
constexpr int kMaxAppendRows = 64;
bool append_fused_ok(const tq_quantizer* q, const tq_kv_cache* c, int n_tokens);
tq_status launch_append_fused(const tq_quantizer* q, tq_kv_cache* c, const void* k_new,
                              const void* v_new, int dtype, int n_tokens, cudaStream_t st);

size_t decode_workspace_bytes(int batch, int n_q_heads, int capacity);
// Fused decode; pdl: launch with programmatic dependent launch (only right after the
// library's own append kernel, which was itself ordered after the query's producer).
tq_status launch_decode(const tq_quantizer* q, const tq_kv_cache* cache, const void* qv,
                        int q_dtype, int n_q_heads, const int32_t* head_map, float sm_scale,
                        void* out, int out_dtype, float* scores, int64_t scores_ld,
                        float* part_out, void* workspace, size_t workspace_bytes, bool pdl,
                        cudaStream_t st);
// The head grouping of a decode over the cache's lengths plus len_add tokens, without
// launching: TQ_EUNSUPPORTED when it needs more head groups than one launch holds.
tq_status check_decode_plan(const tq_quantizer* q, const tq_kv_cache* cache, int n_q_heads,
                            const int32_t* head_map, int len_add);
tq_status set_decode_policy(int policy, int* previous);
tq_status launch_merge_partials(const float* parts, int n_parts, int64_t rows, void* out,
                                int out_dtype, cudaStream_t st);

tq_status launch_decode_noalloc(const tq_quantizer* q, const tq_kv_cache* cache, const void* qv,
                                int q_dtype, int n_q_heads, const int32_t* head_map,
                                float sm_scale, void* out, int out_dtype, float* scores,
                                int64_t scores_ld, cudaStream_t st);

int sm_count(int device);

}  // namespace tq
