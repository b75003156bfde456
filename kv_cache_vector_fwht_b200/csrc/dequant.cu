// Key dequantization (sm_100a): packed planes back to vectors in the original coordinates
// (validate_paper.py dequantize / the reconstruction behind attention_score; tqlite README
// prod.py: x_mse + QJL residual term).
//
//   mse / prod (rotation Pi = H diag(s) / sqrt(d), centroids C at N(0,1) scale):
//     x_hat = Pi^T (n16 C[idx] / sqrt(d)) [+ r16 sqrt(pi/2)/d S^T (2 sigma - 1)],  S = S_rot Pi
//           = s . H w,  w_k = n16 C[idx_k] / d  [+ r16 sqrt(pi/2) / d^1.5 (S_rot^T (2 sigma - 1))_k]
//   grouped: each group g (outliers: 32 channels at b + 1 bits; normals: 96 at b bits) is
//     rotated by 32-point blocks: x_hat[chan] = s . H_32 w,  w = n16_g C_g[idx] / (sqrt(32 d_g)).
//
// One warp per row; lane l holds positions 4l .. 4l + 3 of the rotated vector (grouped: of the
// chain outliers-then-normals, lanes 8k .. 8k + 7 forming 32-point block k). The transform is
// two butterfly stages in registers and 5 (grouped: 3) shuffle stages. prod adds S_rot^T z on
// the CUDA cores with S_rot staged in shared memory (lane l reads columns 4l .. 4l + 3).
#include "tq_device.cuh"
#include "tq_internal.h"

namespace tq {
namespace {

struct DeqArgs {
  const uint8_t* idx;
  const uint8_t* sgn;
  const uint16_t* nrm;
  int64_t n_rows;
  void* out;
  int64_t ld;
  int out_f32;
  const DevTables* tab;
};

// W-bit code j (LSB-first fields) of a row's index bytes.
template <int W>
__device__ __forceinline__ uint32_t code_at(const uint8_t* row, int j) {
  const int bit = j * W;
  return (static_cast<uint32_t>(row[bit >> 3]) >> (bit & 7)) & ((1u << W) - 1u);
}

template <int MODE, int BITS>
__global__ void __launch_bounds__(256) k_dequant_keys(const __grid_constant__ DeqArgs a) {
  constexpr bool PROD = MODE == TQ_MODE_PROD;
  constexpr bool GRP = MODE == TQ_MODE_GROUPED;
  constexpr int MB = PROD ? BITS - 1 : BITS;
  constexpr int W = storage_width_c(MB);                        // mse / prod index width
  constexpr int WO = storage_width_c(BITS + 1), WN = storage_width_c(BITS);  // grouped
  constexpr int IB = GRP ? (32 * WO + 96 * WN) / 8 : kD * W / 8;
  constexpr int NN = PROD || GRP ? 2 : 1;                       // norms per row

  __shared__ __align__(16) __half sS[PROD ? kD * kD : 8];
  const DevTables* __restrict__ tab = a.tab;
  if constexpr (PROD) {
    for (int c = threadIdx.x; c < kD * kD / 8; c += blockDim.x)
      reinterpret_cast<uint4*>(sS)[c] = __ldg(reinterpret_cast<const uint4*>(tab->s_rot) + c);
    __syncthreads();
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + warp; row < a.n_rows;
       row += static_cast<int64_t>(gridDim.x) * 8) {
    const uint8_t* ir = a.idx + row * IB;
    float w[4];
    if constexpr (GRP) {
      const int blk = lane >> 3;                        // 0: outliers, 1..3: normal blocks
      const float n16 = __half2float(__ushort_as_half(a.nrm[row * 2 + (blk ? 1 : 0)]));
      const float sc = n16 * (blk ? 0.10206207261596575f : 0.17677669529663688f) * 0.17677669529663688f;
      // 1/sqrt(96) and 1/sqrt(32) (group dimension), times 1/sqrt(32) (block transform)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int j = 4 * lane + i;
        const uint32_t code = blk ? code_at<WN>(ir + 32 * WO / 8, j - 32) : code_at<WO>(ir, j);
        w[i] = tab->cent[blk ? 1 : 0][code] * sc;
      }
    } else {
      const float n16 = __half2float(__ushort_as_half(a.nrm[row * NN]));
      const float sc = n16 * (1.f / 128.f);
#pragma unroll
      for (int i = 0; i < 4; ++i) w[i] = tab->cent[0][code_at<W>(ir, 4 * lane + i)] * sc;
      if constexpr (PROD) {
        // + r16 sqrt(pi/2) / d^1.5 (S_rot^T z)_k, z_j = +1 if sign bit j is set, else -1
        const float r16 = __half2float(__ushort_as_half(a.nrm[row * 2 + 1]));
        const float cq = r16 * 1.2533141373155002512f / (128.f * 11.313708498984761164f);
        const uint4 sw = __ldg(reinterpret_cast<const uint4*>(a.sgn + row * 16));
        const uint32_t sv[4] = {sw.x, sw.y, sw.z, sw.w};
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
        for (int j = 0; j < kD; ++j) {
          const uint2 s2 = *reinterpret_cast<const uint2*>(sS + j * kD + 4 * lane);
          const float z = ((sv[j >> 5] >> (j & 31)) & 1u) ? 1.f : -1.f;
          acc[0] = fmaf(z, half_lo(s2.x), acc[0]);
          acc[1] = fmaf(z, half_hi(s2.x), acc[1]);
          acc[2] = fmaf(z, half_lo(s2.y), acc[2]);
          acc[3] = fmaf(z, half_hi(s2.y), acc[3]);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) w[i] = fmaf(cq, acc[i], w[i]);
      }
    }
    // x_hat = s . H w: two stages in registers, then across lanes
    fwht_reg<4>(w);
#pragma unroll
    for (int mm = 1; mm < (GRP ? 8 : 32); mm <<= 1) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float other = __shfl_xor_sync(kFull, w[i], mm);
        w[i] = (lane & mm) ? (other - w[i]) : (w[i] + other);
      }
    }
    const uint32_t sb = tab->sign_bits[lane >> 3];
#pragma unroll
    for (int i = 0; i < 4; ++i) w[i] = flip_sign(w[i], sb, (4 * lane + i) & 31);
    if constexpr (GRP) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int ch = tab->chan[4 * lane + i];
        if (a.out_f32) static_cast<float*>(a.out)[row * a.ld + ch] = w[i];
        else static_cast<__nv_bfloat16*>(a.out)[row * a.ld + ch] = __float2bfloat16_rn(w[i]);
      }
    } else if (a.out_f32) {
      *reinterpret_cast<float4*>(static_cast<float*>(a.out) + row * a.ld + 4 * lane) =
          make_float4(w[0], w[1], w[2], w[3]);
    } else {
      const __nv_bfloat162 lo = __floats2bfloat162_rn(w[0], w[1]);
      const __nv_bfloat162 hi = __floats2bfloat162_rn(w[2], w[3]);
      uint2 pk;
      pk.x = *reinterpret_cast<const uint32_t*>(&lo);
      pk.y = *reinterpret_cast<const uint32_t*>(&hi);
      *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(a.out) + row * a.ld + 4 * lane) = pk;
    }
  }
}

template <int MODE, int BITS>
tq_status run_dequant(const DeqArgs& a, cudaStream_t st) {
  int dev = 0;
  cudaGetDevice(&dev);
  const int64_t want = (a.n_rows + 7) / 8;
  const int64_t cap = 8ll * sm_count(dev);
  const int grid = static_cast<int>(want < cap ? want : cap);
  k_dequant_keys<MODE, BITS><<<grid, 256, 0, st>>>(a);
  return cudaGetLastError() == cudaSuccess ? TQ_OK : TQ_ECUDA;
}

}  // namespace

tq_status launch_dequantize_keys(const tq_quantizer* q, tq_key_planes planes, int64_t n_rows,
                                 void* out, int out_dtype, int64_t ld, cudaStream_t st) {
  if (n_rows == 0) return TQ_OK;
  DeqArgs a{planes.idx, planes.signs, planes.norms, n_rows, out, ld, out_dtype == TQ_F32, q->dev};
  switch (q->mode * 8 + q->bits) {
    case TQ_MODE_MSE * 8 + 1: return run_dequant<TQ_MODE_MSE, 1>(a, st);
    case TQ_MODE_MSE * 8 + 2: return run_dequant<TQ_MODE_MSE, 2>(a, st);
    case TQ_MODE_MSE * 8 + 3: return run_dequant<TQ_MODE_MSE, 3>(a, st);
    case TQ_MODE_MSE * 8 + 4: return run_dequant<TQ_MODE_MSE, 4>(a, st);
    case TQ_MODE_PROD * 8 + 2: return run_dequant<TQ_MODE_PROD, 2>(a, st);
    case TQ_MODE_PROD * 8 + 3: return run_dequant<TQ_MODE_PROD, 3>(a, st);
    case TQ_MODE_PROD * 8 + 4: return run_dequant<TQ_MODE_PROD, 4>(a, st);
    case TQ_MODE_GROUPED * 8 + 1: return run_dequant<TQ_MODE_GROUPED, 1>(a, st);
    case TQ_MODE_GROUPED * 8 + 2: return run_dequant<TQ_MODE_GROUPED, 2>(a, st);
    case TQ_MODE_GROUPED * 8 + 3: return run_dequant<TQ_MODE_GROUPED, 3>(a, st);
    default: return TQ_EUNSUPPORTED;
  }
}

}  // namespace tq
