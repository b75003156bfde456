// Fused append of a few new tokens into the packed cache (sm_100a): key quantization
// (mse / prod), value quantization and the length update in one launch
// (TurboQuant bit-packing article, section 5: store.py appends packed tokens).
//
// One warp per new row, lane l holding elements 4l .. 4l + 3. The rotation runs as two
// in-register butterfly stages and five shuffle stages. In prod mode the QJL projection
// S_rot . rho of the (up to) eight rows of a CTA is one tensor-core product: mma.sync
// m16n8k16 with the fp16-exact S_rot as A and the residuals, split into fp16 hi + lo
// halves, as B (fp32 accumulation). Token t of (b, h) goes to cache position
// pos0[b] + t, pos0 being the host-side lengths before the append; every CTA then writes the
// new lengths pos0[b] + n_tokens to the device copy (the same value, no race).
#include "tq_device.cuh"
#include "tq_internal.h"

namespace tq {
namespace {

constexpr int kRowsPerCta = 8;
constexpr int kSStride = 272;  // bytes per staged S_rot / residual row (256 + 16)

struct AppendArgs {
  const void* k;
  const void* v;
  const DevTables* tab;
  uint8_t* idx;
  uint8_t* sgn;
  uint16_t* nrm;
  uint8_t* vq;
  uint16_t* vpar;
  int32_t* len_dev;
  int n_rows, n_kv_heads, n_tokens, capacity, batch;
  int32_t pos0[kMaxAppendBatch];
};

template <int MODE, int BITS, bool F32, int VB>
__global__ void __launch_bounds__(256) k_append(const __grid_constant__ AppendArgs a) {
  constexpr bool PROD = MODE == TQ_MODE_PROD;
  constexpr int MB = PROD ? BITS - 1 : BITS;
  constexpr int NL = 1 << MB;
  constexpr int W = storage_width_c(MB);
  constexpr int IB = kD * W / 8;
  __shared__ __align__(16) uint8_t sS[PROD ? kD * kSStride : 16];
  __shared__ __align__(16) uint8_t sB[PROD ? 2 * kRowsPerCta * kSStride : 16];
  __shared__ float sD[PROD ? kD * (kRowsPerCta + 1) : 1];

  // a decode launched next may start its query-only prologue now (it waits for this grid
  // before it reads the lengths or the cache)
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const DevTables* __restrict__ tab = a.tab;
  if constexpr (PROD) {
    for (int c = threadIdx.x; c < kD * 16; c += blockDim.x) {
      const int r = c >> 4, cc = c & 15;
      cp_async16(sS + r * kSStride + cc * 16,
                 reinterpret_cast<const uint8_t*>(tab->s_rot) + r * 256 + cc * 16, true);
    }
    cp_async_commit();
  }
  const int row = blockIdx.x * kRowsPerCta + warp;
  const bool valid = row < a.n_rows;
  const int t = valid ? row % a.n_tokens : 0;
  const int bh = valid ? row / a.n_tokens : 0;
  const int b = bh / a.n_kv_heads;
  const int64_t orow = static_cast<int64_t>(bh) * a.capacity + (valid ? a.pos0[b] : 0) + t;

  // ---- key: norm, rotation, indices
  float x[4] = {0.f, 0.f, 0.f, 0.f};
  if (valid) {
    if constexpr (F32) load4<true>(static_cast<const float*>(a.k) + static_cast<int64_t>(row) * kD, 4 * lane, x);
    else load4<false>(static_cast<const uint16_t*>(a.k) + static_cast<int64_t>(row) * kD, 4 * lane, x);
  }
  const float n = sqrtf(warp_sum(fmaf(x[0], x[0], fmaf(x[1], x[1], fmaf(x[2], x[2], x[3] * x[3])))));
  const __half n16 = __float2half_rn(n);
  const float n16f = __half2float(n16);
  {
    const uint32_t sw = tab->sign_bits[lane >> 3];
#pragma unroll
    for (int i = 0; i < 4; ++i) x[i] = flip_sign(x[i], sw, (4 * lane + i) & 31);
  }
  fwht_reg<4>(x);
#pragma unroll
  for (int mm = 1; mm < 32; mm <<= 1) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float other = __shfl_xor_sync(kFull, x[i], mm);
      x[i] = (lane & mm) ? (other - x[i]) : (x[i] + other);
    }
  }
  uint32_t code[4];
  float rho[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t id = 0;
    float c = tab->cent[0][0];
#pragma unroll
    for (int k = 0; k < NL - 1; ++k) {
      const float th = tab->thr[0][k];
      const bool gt = x[i] > (n > 0.f ? th * n : th);
      id += gt ? 1u : 0u;
      if constexpr (PROD) c = gt ? tab->cent[0][k + 1] : c;
    }
    code[i] = id;
    rho[i] = fmaf(-n16f, c, x[i]);
  }
  if (valid) {
    if constexpr (W == 2) {
      a.idx[orow * IB + lane] = static_cast<uint8_t>(code[0] | (code[1] << 2) | (code[2] << 4) | (code[3] << 6));
    } else if constexpr (W == 4) {
      reinterpret_cast<uint16_t*>(a.idx + orow * IB)[lane] =
          static_cast<uint16_t>(code[0] | (code[1] << 4) | (code[2] << 8) | (code[3] << 12));
    }
  }
  if constexpr (W == 1) {
    const uint32_t nib = code[0] | (code[1] << 1) | (code[2] << 2) | (code[3] << 3);
    const uint32_t hi = __shfl_down_sync(kFull, nib, 1);
    if (valid && (lane & 1) == 0) a.idx[orow * IB + (lane >> 1)] = static_cast<uint8_t>(nib | (hi << 4));
  }

  if constexpr (!PROD) {
    if (valid && lane == 0) a.nrm[orow] = half_bits(n16);
  } else {
    const float rsq = warp_sum(fmaf(rho[0], rho[0], fmaf(rho[1], rho[1], fmaf(rho[2], rho[2], rho[3] * rho[3]))));
    const __half r16 = __float2half_rn(sqrtf(rsq * (1.f / 128.f)));
    // residual halves for the tensor-core projection (power-of-two scale; sign-preserving)
    float amax = fmaxf(fmaxf(fabsf(rho[0]), fabsf(rho[1])), fmaxf(fabsf(rho[2]), fabsf(rho[3])));
    amax = warp_max(amax);
    const uint32_t ex = (__float_as_uint(amax) >> 23) & 0xffu;
    const float scl = ex >= 12u ? __uint_as_float((264u - ex) << 23) : 1.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float sv = valid ? rho[i] * scl : 0.f;
      const __half hi = __float2half_rn(sv);
      const __half lo = __float2half_rn(sv - __half2float(hi));
      reinterpret_cast<__half*>(sB + warp * kSStride)[4 * lane + i] = hi;
      reinterpret_cast<__half*>(sB + (kRowsPerCta + warp) * kSStride)[4 * lane + i] = lo;
    }
    cp_async_wait<0>();
    __syncthreads();
    {
      // D[j][r] = sum_k S_rot[j][k] rho_r[k]; warp w owns j in [16w, 16w + 16)
      const int g = lane >> 2, tt = lane & 3;
      float c0 = 0.f, c1 = 0.f, c2 = 0.f, c3 = 0.f;
      const uint8_t* arow0 = sS + (16 * warp + g) * kSStride;
      const uint8_t* arow1 = arow0 + 8 * kSStride;
#pragma unroll
      for (int k0 = 0; k0 < kD; k0 += 16) {
        const uint32_t a0 = *reinterpret_cast<const uint32_t*>(arow0 + (k0 + 2 * tt) * 2);
        const uint32_t a1 = *reinterpret_cast<const uint32_t*>(arow1 + (k0 + 2 * tt) * 2);
        const uint32_t a2 = *reinterpret_cast<const uint32_t*>(arow0 + (k0 + 8 + 2 * tt) * 2);
        const uint32_t a3 = *reinterpret_cast<const uint32_t*>(arow1 + (k0 + 8 + 2 * tt) * 2);
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          const uint8_t* bq = sB + (part * kRowsPerCta + g) * kSStride;
          const uint32_t b0 = *reinterpret_cast<const uint32_t*>(bq + (k0 + 2 * tt) * 2);
          const uint32_t b1 = *reinterpret_cast<const uint32_t*>(bq + (k0 + 8 + 2 * tt) * 2);
          asm volatile(
              "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
              "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};\n"
              : "+f"(c0), "+f"(c1), "+f"(c2), "+f"(c3)
              : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
        }
      }
      const int j0 = 16 * warp + g;
      sD[j0 * (kRowsPerCta + 1) + 2 * tt] = c0;
      sD[j0 * (kRowsPerCta + 1) + 2 * tt + 1] = c1;
      sD[(j0 + 8) * (kRowsPerCta + 1) + 2 * tt] = c2;
      sD[(j0 + 8) * (kRowsPerCta + 1) + 2 * tt + 1] = c3;
    }
    __syncthreads();
    uint32_t bits[4];
#pragma unroll
    for (int m = 0; m < 4; ++m)
      bits[m] = __ballot_sync(kFull, sD[(32 * m + lane) * (kRowsPerCta + 1) + warp] >= 0.f);
    if (valid && lane == 0) {
      *reinterpret_cast<uint4*>(a.sgn + orow * 16) = make_uint4(bits[0], bits[1], bits[2], bits[3]);
      *reinterpret_cast<uint32_t*>(a.nrm + orow * 2) =
          static_cast<uint32_t>(half_bits(n16)) | (static_cast<uint32_t>(half_bits(r16)) << 16);
    }
  }

  // ---- value: groups of 32 channels, lane l owns channels 4l .. 4l + 3 (group l / 8)
  if constexpr (VB != 0) {
    constexpr float kLevels = static_cast<float>((1 << VB) - 1);
    float v[4] = {0.f, 0.f, 0.f, 0.f};
    if (valid) {
      if constexpr (F32) load4<true>(static_cast<const float*>(a.v) + static_cast<int64_t>(row) * kD, 4 * lane, v);
      else load4<false>(static_cast<const uint16_t*>(a.v) + static_cast<int64_t>(row) * kD, 4 * lane, v);
    }
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
    uint32_t q[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float tq = __fdiv_rn(__fsub_rn(v[i], mf), sf);
      tq = fminf(fmaxf(rintf(tq), 0.f), kLevels);
      q[i] = sf > 0.f ? static_cast<uint32_t>(tq) : 0u;
    }
    if (valid) {
      if constexpr (VB == 2) {
        a.vq[orow * 32 + lane] = static_cast<uint8_t>(q[0] | (q[1] << 2) | (q[2] << 4) | (q[3] << 6));
      } else {
        reinterpret_cast<uint16_t*>(a.vq + orow * 64)[lane] =
            static_cast<uint16_t>(q[0] | (q[1] << 4) | (q[2] << 8) | (q[3] << 12));
      }
      if ((lane & 7) == 0)
        reinterpret_cast<uint32_t*>(a.vpar + orow * 8)[lane >> 3] =
            static_cast<uint32_t>(half_bits(mn16)) | (static_cast<uint32_t>(half_bits(s16)) << 16);
    }
  }
  if (threadIdx.x < a.batch) a.len_dev[threadIdx.x] = a.pos0[threadIdx.x] + a.n_tokens;
}

template <int MODE, int BITS, bool F32>
tq_status run_append(const AppendArgs& a, int vb, cudaStream_t st) {
  const int grid = (a.n_rows + kRowsPerCta - 1) / kRowsPerCta;
  switch (vb) {
    case 0: k_append<MODE, BITS, F32, 0><<<grid, 256, 0, st>>>(a); break;
    case 2: k_append<MODE, BITS, F32, 2><<<grid, 256, 0, st>>>(a); break;
    default: k_append<MODE, BITS, F32, 4><<<grid, 256, 0, st>>>(a); break;
  }
  return cudaGetLastError() == cudaSuccess ? TQ_OK : TQ_ECUDA;
}

template <bool F32>
tq_status dispatch_append(int mode, int bits, const AppendArgs& a, int vb, cudaStream_t st) {
  switch (mode * 8 + bits) {
    case TQ_MODE_MSE * 8 + 1: return run_append<TQ_MODE_MSE, 1, F32>(a, vb, st);
    case TQ_MODE_MSE * 8 + 2: return run_append<TQ_MODE_MSE, 2, F32>(a, vb, st);
    case TQ_MODE_MSE * 8 + 3: return run_append<TQ_MODE_MSE, 3, F32>(a, vb, st);
    case TQ_MODE_MSE * 8 + 4: return run_append<TQ_MODE_MSE, 4, F32>(a, vb, st);
    case TQ_MODE_PROD * 8 + 2: return run_append<TQ_MODE_PROD, 2, F32>(a, vb, st);
    case TQ_MODE_PROD * 8 + 3: return run_append<TQ_MODE_PROD, 3, F32>(a, vb, st);
    case TQ_MODE_PROD * 8 + 4: return run_append<TQ_MODE_PROD, 4, F32>(a, vb, st);
    default: return TQ_EUNSUPPORTED;
  }
}

}  // namespace

bool append_fused_ok(const tq_quantizer* q, const tq_kv_cache* c, int n_tokens) {
  const int64_t rows = static_cast<int64_t>(c->batch) * c->n_kv_heads * n_tokens;
  return q->mode != TQ_MODE_GROUPED && rows <= kMaxAppendRows && c->batch <= kMaxAppendBatch;
}

tq_status launch_append_fused(const tq_quantizer* q, tq_kv_cache* c, const void* k_new,
                              const void* v_new, int dtype, int n_tokens, cudaStream_t st) {
  AppendArgs a{};
  a.k = k_new;
  a.v = v_new;
  a.tab = q->dev;
  a.idx = c->keys.idx;
  a.sgn = c->keys.signs;
  a.nrm = c->keys.norms;
  a.vq = c->values.q;
  a.vpar = c->values.params;
  a.len_dev = c->len_dev;
  a.n_rows = c->batch * c->n_kv_heads * n_tokens;
  a.n_kv_heads = c->n_kv_heads;
  a.n_tokens = n_tokens;
  a.capacity = c->capacity;
  a.batch = c->batch;
  for (int b = 0; b < c->batch; ++b) a.pos0[b] = c->len_host[b];
  return dtype == TQ_F32 ? dispatch_append<true>(q->mode, q->bits, a, c->value_bits, st)
                         : dispatch_append<false>(q->mode, q->bits, a, c->value_bits, st);
}

}  // namespace tq
