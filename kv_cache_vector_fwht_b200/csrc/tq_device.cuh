// Device helpers shared by the libtq kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

namespace tq {

constexpr unsigned kFull = 0xffffffffu;

__host__ __device__ constexpr int storage_width_c(int bits) {
  return bits == 1 ? 1 : (bits == 2 ? 2 : 4);
}

// Eight consecutive row elements as fp32: bf16 rows take one 16-byte load, fp32 rows two.
template <bool F32>
__device__ __forceinline__ void load8(const void* row, int e, float (&v)[8]) {
  if constexpr (F32) {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(row) + e);
    const float4 a = __ldg(p), b = __ldg(p + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  } else {
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(
        static_cast<const uint16_t*>(row) + e));
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(ws[i] << 16);
      v[2 * i + 1] = __uint_as_float(ws[i] & 0xffff0000u);
    }
  }
}

// Four consecutive elements as fp32 (bf16: one 8-byte load, fp32: one 16-byte load).
template <bool F32>
__device__ __forceinline__ void load4(const void* row, int e, float (&v)[4]) {
  if constexpr (F32) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(static_cast<const float*>(row) + e));
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  } else {
    const uint2 w = __ldg(reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(row) + e));
    v[0] = __uint_as_float(w.x << 16);
    v[1] = __uint_as_float(w.x & 0xffff0000u);
    v[2] = __uint_as_float(w.y << 16);
    v[3] = __uint_as_float(w.y & 0xffff0000u);
  }
}

// x * s_j where bit `bit` of `word` set means s_j = -1 (a sign-bit flip, exact).
__device__ __forceinline__ float flip_sign(float x, uint32_t word, int bit) {
  return __uint_as_float(__float_as_uint(x) ^ ((word << (31 - bit)) & 0x80000000u));
}

// In-register Walsh-Hadamard butterflies (Sylvester order, unnormalised) on N values.
template <int N>
__device__ __forceinline__ void fwht_reg(float* v) {
#pragma unroll
  for (int h = 1; h < N; h <<= 1) {
#pragma unroll
    for (int i = 0; i < N; ++i) {
      if ((i & h) == 0) {
        const float a = v[i], b = v[i + h];
        v[i] = a + b;
        v[i + h] = a - b;
      }
    }
  }
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, m));
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) v += __shfl_xor_sync(kFull, v, m);
  return v;
}

__device__ __forceinline__ uint16_t half_bits(__half h) { return __half_as_ushort(h); }

__device__ __forceinline__ float half_lo(uint32_t w) {
  return __half2float(__ushort_as_half(static_cast<uint16_t>(w & 0xffffu)));
}
__device__ __forceinline__ float half_hi(uint32_t w) {
  return __half2float(__ushort_as_half(static_cast<uint16_t>(w >> 16)));
}

// cp.async 16-byte global->shared copy (L2 only), zero-filling when !pred.
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, bool pred) {
  const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  const int n = pred ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem), "r"(n));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

}  // namespace tq
