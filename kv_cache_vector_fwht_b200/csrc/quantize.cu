// Key and value quantization kernels (sm_100a).
//
// Keys (tqlite README: mse.py, prod.py, grouped.py; Implementing TurboQuant (part 5),
// algorithm overview; TurboQuant bit-packing article sections 2-4):
//   n = ||x||, y = H (s . x) (unnormalised Sylvester Hadamard after the sign flips, so
//   Pi x = y / sqrt(d)), idx_j = #{k : y_j > t_k n} (the decision u_j = (Pi x)_j / n > t_k /
//   sqrt(d) with N(0,1)-scale edges t_k), packed lowest bits first; prod adds
//   rho = y - n16 C[idx] (= sqrt(d) Pi r), ||r|| = ||rho|| / sqrt(d) and the QJL bits
//   [(S_rot rho)_j >= 0] (= [(S r)_j >= 0] with S = S_rot Pi).
// Values: per 32-channel group, fp16 (min, scale) and codes rint((v - mn16) / s16) computed
// with IEEE fp32 subtract and divide.
//
// Thread layout of the full-width key kernel: two lanes per row. Lane h of a row loads the
// whole row, forms a = (s.x)[0:64], b = (s.x)[64:128] and keeps a + b (h = 0) or a - b
// (h = 1): the first butterfly stage of H_128 = [[H_64, H_64], [H_64, -H_64]]. The remaining
// six stages run in registers, so lane h ends with coordinates [64h, 64h + 64) of y.
#include <cfloat>
#include <cstddef>

#include "tq_device.cuh"
#include "tq_internal.h"

namespace tq {
namespace {

struct KeyArgs {
  const void* x;
  int64_t n_rows;
  int64_t ld;
  const DevTables* tab;
  uint8_t* idx;
  uint8_t* sgn;
  uint16_t* nrm;
  RowMap map;
};

__device__ __forceinline__ int64_t out_row(const RowMap& m, int64_t r) {
  if (m.len == nullptr) return r;
  const int t = static_cast<int>(r % m.n_tokens);
  const int64_t bh = r / m.n_tokens;
  const int b = static_cast<int>(bh / m.n_kv_heads);
  return bh * m.capacity + m.len[b] + t;
}

constexpr int kRhoStride = 129;  // floats per staged residual row (bank spread)

// ---------------------------------------------------------------------------------------
// mse / prod keys, d = 128
// ---------------------------------------------------------------------------------------
template <int MODE, int BITS, bool F32>
__global__ void __launch_bounds__(256) k_keys_full(KeyArgs a) {
  constexpr int MB = MODE == TQ_MODE_PROD ? BITS - 1 : BITS;  // codebook width
  constexpr int NL = 1 << MB;
  constexpr int W = storage_width_c(MB);
  constexpr int IB = kD * W / 8;      // index bytes per row
  constexpr int HW = IB / 8;          // 32-bit words per lane half
  constexpr bool PROD = MODE == TQ_MODE_PROD;

  extern __shared__ __align__(16) float smem[];
  float* sST = smem;                          // prod: S_rot^T in fp32, [i][j] = S_rot[j][i]
  float* sRho = smem + (PROD ? kD * kD : 0);  // prod: [warps][16 rows][kRhoStride]

  const DevTables* __restrict__ tab = a.tab;
  float thr[NL - 1], cen[NL];
#pragma unroll
  for (int k = 0; k < NL - 1; ++k) thr[k] = tab->thr[0][k];
#pragma unroll
  for (int k = 0; k < NL; ++k) cen[k] = tab->cent[0][k];
  uint32_t sb[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) sb[k] = tab->sign_bits[k];

  if constexpr (PROD) {
    // 16-byte loads of 8 fp16 entries each (a small batch runs 2-warp blocks, for which
    // element-wise loads made this staging most of the kernel's time)
    static_assert(offsetof(DevTables, s_rot_t) % 16 == 0, "16-byte aligned S_rot^T");
    const uint4* src = reinterpret_cast<const uint4*>(tab->s_rot_t);
#pragma unroll 4
    for (int e8 = threadIdx.x; e8 < kD * kD / 8; e8 += blockDim.x) {
      const uint4 v = __ldg(src + e8);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
      float f[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 p = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
        f[2 * i] = p.x;
        f[2 * i + 1] = p.y;
      }
      float4* d = reinterpret_cast<float4*>(sST + 8 * e8);
      d[0] = make_float4(f[0], f[1], f[2], f[3]);
      d[1] = make_float4(f[4], f[5], f[6], f[7]);
    }
    __syncthreads();
  }

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarps = static_cast<int>(blockDim.x >> 5);
  const int hf = lane & 1, rl = lane >> 1;
  const uint32_t hmask = static_cast<uint32_t>(hf) << 31;
  const int64_t n_groups = (a.n_rows + 15) / 16;

  for (int64_t g = static_cast<int64_t>(blockIdx.x) * nwarps + warp; g < n_groups;
       g += static_cast<int64_t>(gridDim.x) * nwarps) {
    const int64_t row = g * 16 + rl;
    const bool valid = row < a.n_rows;
    const int64_t src = valid ? row : a.n_rows - 1;
    const void* prow = F32 ? static_cast<const void*>(static_cast<const float*>(a.x) + src * a.ld)
                           : static_cast<const void*>(static_cast<const uint16_t*>(a.x) + src * a.ld);

    float u[64];
    float ss = 0.f;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      float xl[8], xh[8];
      load8<F32>(prow, 8 * c, xl);
      load8<F32>(prow, 64 + 8 * c, xh);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int j = 8 * c + i;
        const float mine = hf ? xh[i] : xl[i];
        ss = fmaf(mine, mine, ss);
        const float lo = flip_sign(xl[i], sb[j >> 5], j & 31);
        const float hi = __uint_as_float(__float_as_uint(flip_sign(xh[i], sb[(j + 64) >> 5],
                                                                   (j + 64) & 31)) ^ hmask);
        u[j] = lo + hi;
      }
    }
    const float nsq = ss + __shfl_xor_sync(kFull, ss, 1);
    const float n = sqrtf(nsq);
    const __half n16 = __float2half_rn(n);
    const float n16f = __half2float(n16);

    fwht_reg<64>(u);

    float T[NL - 1];
#pragma unroll
    for (int k = 0; k < NL - 1; ++k) T[k] = n > 0.f ? thr[k] * n : thr[k];

    uint32_t pk[HW];
#pragma unroll
    for (int w = 0; w < HW; ++w) pk[w] = 0u;
    float rss = 0.f;
#pragma unroll
    for (int j = 0; j < 64; ++j) {
      const float y = u[j];
      uint32_t id = 0;
      float c = cen[0];
#pragma unroll
      for (int k = 0; k < NL - 1; ++k) {
        const bool gt = y > T[k];
        id += gt ? 1u : 0u;
        if constexpr (PROD) c = gt ? cen[k + 1] : c;
      }
      pk[(j * W) >> 5] |= id << ((j * W) & 31);
      if constexpr (PROD) {
        const float r = fmaf(-n16f, c, y);
        u[j] = r;
        rss = fmaf(r, r, rss);
      }
    }

    const int64_t orow = valid ? out_row(a.map, row) : 0;
    if (valid) {
      uint8_t* dst = a.idx + orow * IB + hf * (IB / 2);
      if constexpr (HW == 2) {
        *reinterpret_cast<uint2*>(dst) = make_uint2(pk[0], pk[1]);
      } else {
#pragma unroll
        for (int w = 0; w < HW; w += 4)
          *reinterpret_cast<uint4*>(dst + 4 * w) = make_uint4(pk[w], pk[w + 1], pk[w + 2], pk[w + 3]);
      }
    }

    if constexpr (!PROD) {
      if (valid && hf == 0) a.nrm[orow] = half_bits(n16);
    } else {
      const float rsq = rss + __shfl_xor_sync(kFull, rss, 1);
      const __half r16 = __float2half_rn(sqrtf(rsq * (1.f / 128.f)));
      float* my = sRho + (warp * 16 + rl) * kRhoStride;
#pragma unroll
      for (int j = 0; j < 64; ++j) my[hf * 64 + j] = u[j];
      __syncwarp();
      // packed fp32x2 multiply-adds: the same rounding per element as scalar ones
      uint64_t acc2[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) acc2[j] = 0ull;
#pragma unroll 2
      for (int i = 0; i < kD; ++i) {
        const float ri = my[i];
        const uint64_t ri2 = pk2(ri, ri);
        const ulonglong2* srow = reinterpret_cast<const ulonglong2*>(sST + i * kD + hf * 64);
#pragma unroll
        for (int q4 = 0; q4 < 16; ++q4) {
          const ulonglong2 sv = srow[q4];
          acc2[2 * q4] = fma2(sv.x, ri2, acc2[2 * q4]);
          acc2[2 * q4 + 1] = fma2(sv.y, ri2, acc2[2 * q4 + 1]);
        }
      }
      float acc[64];
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const float2 v = up2(acc2[j]);
        acc[2 * j] = v.x;
        acc[2 * j + 1] = v.y;
      }
      uint32_t sg0 = 0u, sg1 = 0u;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        sg0 |= (acc[j] >= 0.f ? 1u : 0u) << j;
        sg1 |= (acc[32 + j] >= 0.f ? 1u : 0u) << j;
      }
      if (valid) {
        *reinterpret_cast<uint2*>(a.sgn + orow * 16 + hf * 8) = make_uint2(sg0, sg1);
        if (hf == 0) {
          const uint32_t nn = static_cast<uint32_t>(half_bits(n16)) |
                              (static_cast<uint32_t>(half_bits(r16)) << 16);
          *reinterpret_cast<uint32_t*>(a.nrm + orow * 2) = nn;
        }
      }
      __syncwarp();
    }
  }
}

// ---------------------------------------------------------------------------------------
// grouped keys: 32 outlier channels at BITS+1 bits, 96 normal channels at BITS bits.
// Four lanes per row; lane k owns 32-channel block k (k = 0: outlier group, k = 1..3: the
// normal group's three FWHT-32 blocks).
// ---------------------------------------------------------------------------------------
template <int BITS, bool F32>
__global__ void __launch_bounds__(256) k_keys_grouped(KeyArgs a) {
  constexpr int BO = BITS + 1, BN = BITS;
  constexpr int WO = storage_width_c(BO), WN = storage_width_c(BN);
  constexpr int OB = 32 * WO / 8, NB = 32 * WN / 8;
  constexpr int IB = OB + 3 * NB;
  constexpr int NLO = 1 << BO, NLN = 1 << BN;

  __shared__ float sRow[8][8][kRhoStride];
  __shared__ uint8_t sChan[kD];
  const DevTables* __restrict__ tab = a.tab;
  for (int e = threadIdx.x; e < kD; e += blockDim.x) sChan[e] = tab->chan[e];
  __syncthreads();

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int k = lane & 3, rl = lane >> 2;
  const uint32_t sbk = tab->sign_bits[k];
  float thrO[NLO - 1], thrN[NLN - 1];
#pragma unroll
  for (int i = 0; i < NLO - 1; ++i) thrO[i] = tab->thr[0][i];
#pragma unroll
  for (int i = 0; i < NLN - 1; ++i) thrN[i] = tab->thr[1][i];

  const int64_t n_groups = (a.n_rows + 7) / 8;
  for (int64_t g = static_cast<int64_t>(blockIdx.x) * 8 + warp; g < n_groups;
       g += static_cast<int64_t>(gridDim.x) * 8) {
    // stage 8 rows: lane loads elements [4 lane, 4 lane + 4) of each
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      int64_t row = g * 8 + r;
      if (row >= a.n_rows) row = a.n_rows - 1;
      const void* prow = F32 ? static_cast<const void*>(static_cast<const float*>(a.x) + row * a.ld)
                             : static_cast<const void*>(static_cast<const uint16_t*>(a.x) + row * a.ld);
      float v[4];
      load4<F32>(prow, 4 * lane, v);
#pragma unroll
      for (int i = 0; i < 4; ++i) sRow[warp][r][4 * lane + i] = v[i];
    }
    __syncwarp();
    const int64_t row = g * 8 + rl;
    const bool valid = row < a.n_rows;

    float x[32];
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const float xi = sRow[warp][rl][sChan[32 * k + i]];
      ss = fmaf(xi, xi, ss);
      x[i] = flip_sign(xi, sbk, i);
    }
    // norms: outlier block alone; normal group = blocks 1..3 of the same row
    const float s1 = __shfl_sync(kFull, ss, (lane & ~3) + 1);
    const float s2 = __shfl_sync(kFull, ss, (lane & ~3) + 2);
    const float s3 = __shfl_sync(kFull, ss, (lane & ~3) + 3);
    const float n = k == 0 ? sqrtf(ss) : sqrtf(s1 + s2 + s3);
    const __half n16 = __float2half_rn(n);

    fwht_reg<32>(x);

    uint8_t* dst = a.idx + (valid ? out_row(a.map, row) : 0) * IB;
    if (k == 0) {
      float T[NLO - 1];
#pragma unroll
      for (int i = 0; i < NLO - 1; ++i) T[i] = n > 0.f ? thrO[i] * n : thrO[i];
      uint32_t pk[OB / 4];
#pragma unroll
      for (int w = 0; w < OB / 4; ++w) pk[w] = 0u;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        uint32_t id = 0;
#pragma unroll
        for (int t = 0; t < NLO - 1; ++t) id += x[j] > T[t] ? 1u : 0u;
        pk[(j * WO) >> 5] |= id << ((j * WO) & 31);
      }
      if (valid) {
#pragma unroll
        for (int w = 0; w < OB / 4; ++w) reinterpret_cast<uint32_t*>(dst)[w] = pk[w];
      }
    } else {
      const float ns = n * 0.57735026918962576f;  // sqrt(32 / 96)
      float T[NLN - 1];
#pragma unroll
      for (int i = 0; i < NLN - 1; ++i) T[i] = n > 0.f ? thrN[i] * ns : thrN[i];
      uint32_t pk[NB / 4];
#pragma unroll
      for (int w = 0; w < NB / 4; ++w) pk[w] = 0u;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        uint32_t id = 0;
#pragma unroll
        for (int t = 0; t < NLN - 1; ++t) id += x[j] > T[t] ? 1u : 0u;
        pk[(j * WN) >> 5] |= id << ((j * WN) & 31);
      }
      if (valid) {
        uint32_t* d32 = reinterpret_cast<uint32_t*>(dst + OB + (k - 1) * NB);
#pragma unroll
        for (int w = 0; w < NB / 4; ++w) d32[w] = pk[w];
      }
    }
    if (valid && k < 2) a.nrm[(valid ? out_row(a.map, row) : 0) * 2 + k] = half_bits(n16);
    __syncwarp();
  }
}

// ---------------------------------------------------------------------------------------
// values: one warp per row, lane l owns channels 4l..4l+3 (group l / 8)
// ---------------------------------------------------------------------------------------
struct ValArgs {
  const void* v;
  int64_t n_rows;
  int64_t ld;
  uint8_t* q;
  uint16_t* par;
  RowMap map;
};

template <int VB, bool F32>
__global__ void __launch_bounds__(256) k_values(ValArgs a) {
  constexpr float kLevels = static_cast<float>((1 << VB) - 1);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + warp; row < a.n_rows;
       row += static_cast<int64_t>(gridDim.x) * 8) {
    const void* prow = F32 ? static_cast<const void*>(static_cast<const float*>(a.v) + row * a.ld)
                           : static_cast<const void*>(static_cast<const uint16_t*>(a.v) + row * a.ld);
    float v[4];
    load4<F32>(prow, 4 * lane, v);
    float mn = fminf(fminf(v[0], v[1]), fminf(v[2], v[3]));
    float mx = fmaxf(fmaxf(v[0], v[1]), fmaxf(v[2], v[3]));
#pragma unroll
    for (int m = 1; m <= 4; m <<= 1) {
      mn = fminf(mn, __shfl_xor_sync(kFull, mn, m));
      mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, m));
    }
    const float scale = __fdiv_rn(__fsub_rn(mx, mn), kLevels);
    const __half s16 = __float2half_rn(scale);
    const __half mn16 = __float2half_rn(mn);
    const float sf = __half2float(s16), mf = __half2float(mn16);
    uint32_t code[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float t = __fdiv_rn(__fsub_rn(v[i], mf), sf);
      t = fminf(fmaxf(rintf(t), 0.f), kLevels);
      code[i] = sf > 0.f ? static_cast<uint32_t>(t) : 0u;
    }
    const int64_t orow = out_row(a.map, row);
    if constexpr (VB == 2) {
      a.q[orow * 32 + lane] =
          static_cast<uint8_t>(code[0] | (code[1] << 2) | (code[2] << 4) | (code[3] << 6));
    } else {
      reinterpret_cast<uint16_t*>(a.q + orow * 64)[lane] =
          static_cast<uint16_t>(code[0] | (code[1] << 4) | (code[2] << 8) | (code[3] << 12));
    }
    if ((lane & 7) == 0) {
      reinterpret_cast<uint32_t*>(a.par + orow * 8)[lane >> 3] =
          static_cast<uint32_t>(half_bits(mn16)) | (static_cast<uint32_t>(half_bits(s16)) << 16);
    }
  }
}

__global__ void k_advance_len(int32_t* len, int batch, int n) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < batch) len[b] += n;
}

template <typename K>
int grid_for(K kernel, int block, size_t smem, int64_t work_items_per_block, int64_t items) {
  int dev = 0, per_sm = 1;
  cudaGetDevice(&dev);
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, block, smem);
  if (per_sm < 1) per_sm = 1;
  const int64_t want = (items + work_items_per_block - 1) / work_items_per_block;
  const int64_t cap = static_cast<int64_t>(sm_count(dev)) * per_sm;
  return static_cast<int>(want < cap ? (want < 1 ? 1 : want) : cap);
}

template <int MODE, int BITS, bool F32>
tq_status run_full(const KeyArgs& a, cudaStream_t st) {
  constexpr bool PROD = MODE == TQ_MODE_PROD;
  // 8 warps (128 rows) per block; inputs too small to give every SM a block take 2-warp
  // blocks (32 rows each, 4x the blocks)
  int dev = 0;
  cudaGetDevice(&dev);
  const int warps = a.n_rows < static_cast<int64_t>(sm_count(dev)) * 128 ? 2 : 8;
  const size_t smem = PROD ? (kD * kD + warps * 16 * kRhoStride) * sizeof(float) : 0;
  auto kern = k_keys_full<MODE, BITS, F32>;
  static bool attr_set = false;
  if (PROD && !attr_set) {
    const size_t smem_max = (kD * kD + 8 * 16 * kRhoStride) * sizeof(float);
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem_max)) != cudaSuccess)
      return TQ_ECUDA;
    attr_set = true;
  }
  const int grid = grid_for(kern, 32 * warps, smem, warps * 16, a.n_rows);
  kern<<<grid, 32 * warps, smem, st>>>(a);
  return cudaGetLastError() == cudaSuccess ? TQ_OK : TQ_ECUDA;
}

template <int BITS, bool F32>
tq_status run_grouped(const KeyArgs& a, cudaStream_t st) {
  auto kern = k_keys_grouped<BITS, F32>;
  const int grid = grid_for(kern, 256, 0, 8 * 8, a.n_rows);
  kern<<<grid, 256, 0, st>>>(a);
  return cudaGetLastError() == cudaSuccess ? TQ_OK : TQ_ECUDA;
}

template <bool F32>
tq_status dispatch_keys(int mode, int bits, const KeyArgs& a, cudaStream_t st) {
  switch (mode * 8 + bits) {
    case TQ_MODE_MSE * 8 + 1: return run_full<TQ_MODE_MSE, 1, F32>(a, st);
    case TQ_MODE_MSE * 8 + 2: return run_full<TQ_MODE_MSE, 2, F32>(a, st);
    case TQ_MODE_MSE * 8 + 3: return run_full<TQ_MODE_MSE, 3, F32>(a, st);
    case TQ_MODE_MSE * 8 + 4: return run_full<TQ_MODE_MSE, 4, F32>(a, st);
    case TQ_MODE_PROD * 8 + 2: return run_full<TQ_MODE_PROD, 2, F32>(a, st);
    case TQ_MODE_PROD * 8 + 3: return run_full<TQ_MODE_PROD, 3, F32>(a, st);
    case TQ_MODE_PROD * 8 + 4: return run_full<TQ_MODE_PROD, 4, F32>(a, st);
    case TQ_MODE_GROUPED * 8 + 1: return run_grouped<1, F32>(a, st);
    case TQ_MODE_GROUPED * 8 + 2: return run_grouped<2, F32>(a, st);
    case TQ_MODE_GROUPED * 8 + 3: return run_grouped<3, F32>(a, st);
    default: return TQ_EUNSUPPORTED;
  }
}

}  // namespace

tq_status launch_quantize_keys(const tq_quantizer* q, const void* x, int dtype, int64_t n_rows,
                               int64_t ld, tq_key_planes out, RowMap map, cudaStream_t st) {
  if (n_rows == 0) return TQ_OK;
  if (keys_tc_ok(q, dtype)) return launch_keys_tc(q, x, n_rows, ld, out, map, st);
  KeyArgs a{x, n_rows, ld, q->dev, out.idx, out.signs, out.norms, map};
  return dtype == TQ_F32 ? dispatch_keys<true>(q->mode, q->bits, a, st)
                         : dispatch_keys<false>(q->mode, q->bits, a, st);
}

tq_status launch_quantize_values(const void* v, int dtype, int64_t n_rows, int64_t ld, int bits,
                                 tq_value_planes out, RowMap map, cudaStream_t st) {
  if (n_rows == 0) return TQ_OK;
  ValArgs a{v, n_rows, ld, out.q, out.params, map};
  const bool f32 = dtype == TQ_F32;
  int grid;
  if (bits == 2 && f32) {
    grid = grid_for(k_values<2, true>, 256, 0, 8, n_rows);
    k_values<2, true><<<grid, 256, 0, st>>>(a);
  } else if (bits == 2) {
    grid = grid_for(k_values<2, false>, 256, 0, 8, n_rows);
    k_values<2, false><<<grid, 256, 0, st>>>(a);
  } else if (f32) {
    grid = grid_for(k_values<4, true>, 256, 0, 8, n_rows);
    k_values<4, true><<<grid, 256, 0, st>>>(a);
  } else {
    grid = grid_for(k_values<4, false>, 256, 0, 8, n_rows);
    k_values<4, false><<<grid, 256, 0, st>>>(a);
  }
  return cudaGetLastError() == cudaSuccess ? TQ_OK : TQ_ECUDA;
}

tq_status launch_advance_len(int32_t* len, int batch, int n, cudaStream_t st) {
  k_advance_len<<<(batch + 127) / 128, 128, 0, st>>>(len, batch, n);
  return cudaGetLastError() == cudaSuccess ? TQ_OK : TQ_ECUDA;
}

}  // namespace tq
