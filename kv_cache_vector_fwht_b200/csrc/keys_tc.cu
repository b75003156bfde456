// prod-mode key quantization of bf16 rows with the QJL projection on the 5th-generation
// tensor cores (sm_100a: tcgen05.mma, operands and accumulator in tensor memory / shared
// memory).
//
// What is computed (tqlite README: rotation.py, codebook.py, prod.py; Implementing TurboQuant
// (part 5), algorithm overview; TurboQuant bit-packing article sections 2-4), per row x:
//   n = ||x||, y = H (s . x) (unnormalised Sylvester Hadamard, so Pi x = y / sqrt(d)),
//   idx_j = #{k : y_j > t_k n}, rho = y - n16 C[idx] (= sqrt(d) Pi r), ||r|| = ||rho|| / sqrt(d),
//   QJL bits [(S_rot rho)_j >= 0] (= [(S r)_j >= 0] with S = S_rot Pi).
//
// Work split. A CTA of four warps owns a tile of 128 rows: thread i owns row i of the tile,
// which is also lane i of the tensor-memory accumulator. Rows arrive in shared memory by
// bulk copies (double-buffered, one tile ahead); the norm, the rotation (seven butterfly
// stages in registers), the codebook decisions and the residual run on the CUDA cores. The
// residual, scaled by a power of two and split into fp16 hi + lo halves, is written to tensor
// memory as the A operand (128 x 256, K = hi then lo); S_rot, fp16-exact, sits in shared
// memory as the B operand. Sixteen m128 n128 k16 MMAs accumulate D = [hi | lo] [S | S]^T in
// fp32 (hi and lo products are exact in fp32, so D carries the fp32 accuracy of S_rot rho).
// The sign bits of D are taken while the next tile is rotated.
//
// Registers hold the row as 64 fp32 pairs (y_p, y_{p + 64}); the K order of both operands is
// permuted to match (k' = 2p holds element p, k' = 2p + 1 element p + 64), which leaves the
// product unchanged.
#include "tq_device.cuh"
#include "tq_internal.h"

namespace tq {
namespace {

constexpr int kTile = 128;             // rows per tile = MMA M = TMEM lanes
constexpr int kXStride = 272;          // bytes per staged row (256 + 16: conflict-free reads)
constexpr int kXBuf = kTile * kXStride;
constexpr int kBBytes = kD * kD * 2;   // S_rot operand
constexpr int kSmemBytes = kBBytes + 2 * kXBuf + 256;
constexpr uint32_t kTmemCols = 256;    // D: columns [0, 128); A: hi [128, 192), lo [192, 256)
constexpr uint64_t kWaitNs = 2000000000ull;

struct TcKeyArgs {
  const uint16_t* x;
  int64_t n_rows;
  int64_t ld;
  int64_t n_tiles;
  const DevTables* tab;
  uint8_t* idx;
  uint8_t* sgn;
  uint16_t* nrm;
  RowMap map;
  int* err;
};

__device__ __forceinline__ int64_t out_row_tc(const RowMap& m, int64_t r) {
  if (m.len == nullptr) return r;
  const int t = static_cast<int>(r % m.n_tokens);
  const int64_t bh = r / m.n_tokens;
  const int b = static_cast<int>(bh / m.n_kv_heads);
  return bh * m.capacity + m.len[b] + t;
}

__device__ __forceinline__ uint32_t h2_bits(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Issue the bulk copies of local tile k into buffer k & 1 (called by warp 0).
__device__ __forceinline__ void issue_tile(const TcKeyArgs& a, uint8_t* sX, uint64_t* bar,
                                           int64_t tile, int lane) {
  const int64_t r0 = tile * kTile;
  const int nv = static_cast<int>(a.n_rows - r0 < kTile ? a.n_rows - r0 : kTile);
  if (lane == 0) mbar_expect_tx(bar, static_cast<uint32_t>(nv) * 256u);
  __syncwarp();
  for (int r = lane; r < nv; r += 32)
    bulk_g2s(sX + r * kXStride, a.x + (r0 + r) * a.ld, 256u, bar);
}

// Sign bits [D_j >= 0] of this thread's accumulator row, stored as the row's 16-byte plane.
__device__ __forceinline__ void store_signs(const TcKeyArgs& a, uint32_t tlane, bool valid,
                                            int64_t row) {
  uint32_t sg[4] = {0u, 0u, 0u, 0u};
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    uint32_t d[16];
    tmem_ld16(tlane + 16 * q, d);
    tmem_ld_wait();
#pragma unroll
    for (int i = 0; i < 16; ++i)
      sg[q >> 1] |= (__uint_as_float(d[i]) >= 0.f ? 1u : 0u) << (16 * (q & 1) + i);
  }
  if (valid)
    *reinterpret_cast<uint4*>(a.sgn + out_row_tc(a.map, row) * 16) =
        make_uint4(sg[0], sg[1], sg[2], sg[3]);
}

template <int MB>
__global__ void __launch_bounds__(128, 2) k_keys_prod_tc(const __grid_constant__ TcKeyArgs a) {
  constexpr int NL = 1 << MB;
  constexpr int W = storage_width_c(MB);
  constexpr int IB = kD * W / 8;  // index bytes per row
  constexpr int NW = IB / 4;      // index words per row

  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* sB = smem;
  uint8_t* sX = smem + kBBytes;
  uint32_t* sMask = reinterpret_cast<uint32_t*>(smem + kBBytes + 2 * kXBuf);
  __shared__ __align__(8) uint64_t bar_x[2];
  __shared__ __align__(8) uint64_t bar_mma;
  __shared__ uint32_t tslot;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const DevTables* __restrict__ tab = a.tab;
  const int64_t grid = gridDim.x;
  const int64_t n_local = a.n_tiles > blockIdx.x ? (a.n_tiles - blockIdx.x + grid - 1) / grid : 0;

  if (warp == 0) {
    tmem_alloc(&tslot, kTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&bar_x[0], 1);
    mbar_init(&bar_x[1], 1);
    mbar_init(&bar_mma, 1);
    fence_mbar_init();
  }
  // B operand: S_rot with the permuted K order, canonical K-major no-swizzle layout
  // (8-row x 16-byte core matrices; K-adjacent core matrices 128 B apart, 8-row groups 2 KB).
  for (int c = tid; c < kD * 16; c += blockDim.x) {
    const int j = c >> 4, kc = c & 15;
    const __half* srow = tab->s_rot + j * kD;
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int p = 4 * kc + i;
      w[i] = static_cast<uint32_t>(__half_as_ushort(srow[p])) |
             (static_cast<uint32_t>(__half_as_ushort(srow[p + 64])) << 16);
    }
    *reinterpret_cast<uint4*>(sB + (j >> 3) * 2048 + kc * 128 + (j & 7) * 16) =
        make_uint4(w[0], w[1], w[2], w[3]);
  }
  // sign masks for bf16 pairs: word q flips elements 2q (bit 15) and 2q + 1 (bit 31)
  if (tid < 64) {
    const int j = 2 * tid;
    const uint32_t b0 = (tab->sign_bits[j >> 5] >> (j & 31)) & 1u;
    const uint32_t b1 = (tab->sign_bits[(j + 1) >> 5] >> ((j + 1) & 31)) & 1u;
    sMask[tid] = (b0 << 15) | (b1 << 31);
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = tslot;
  const uint32_t tlane = tbase + (static_cast<uint32_t>(warp * 32) << 16);

  float thr[NL - 1], cen[NL];
#pragma unroll
  for (int k = 0; k < NL - 1; ++k) thr[k] = tab->thr[0][k];
#pragma unroll
  for (int k = 0; k < NL; ++k) cen[k] = tab->cent[0][k];

  if (warp == 0) {
    if (n_local > 0) issue_tile(a, sX, &bar_x[0], blockIdx.x, lane);
    if (n_local > 1) issue_tile(a, sX + kXBuf, &bar_x[1], blockIdx.x + grid, lane);
  }

  constexpr uint32_t idesc = umma_idesc_f16(kTile, kD);
  bool failed = false;
  int64_t prev_row = -1;  // global row of this thread in the previous tile (-1: none)
  bool prev_valid = false;

  for (int64_t k = 0; k < n_local; ++k) {
    const int b = static_cast<int>(k & 1);
    const uint32_t ph = static_cast<uint32_t>((k >> 1) & 1);
    const int64_t tile = blockIdx.x + k * grid;
    if (!__syncthreads_and(mbar_wait_ns(&bar_x[b], ph, kWaitNs))) {
      failed = true;
      break;
    }
    const int64_t row = tile * kTile + tid;
    const bool valid = row < a.n_rows;

    // ---- load the row, flip signs, norm; pairs P[p] = (x_p, x_{p+64})
    uint64_t P[64];
    float ss;
    {
      const uint8_t* xr = sX + b * kXBuf + tid * kXStride;
      uint32_t wl[32], wh[32];  // bf16 pairs of elements [0, 64) and [64, 128)
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint4 u0 = *reinterpret_cast<const uint4*>(xr + 16 * c);
        const uint4 u1 = *reinterpret_cast<const uint4*>(xr + 128 + 16 * c);
        const uint4 m0 = *reinterpret_cast<const uint4*>(sMask + 4 * c);
        const uint4 m1 = *reinterpret_cast<const uint4*>(sMask + 32 + 4 * c);
        wl[4 * c + 0] = u0.x ^ m0.x; wl[4 * c + 1] = u0.y ^ m0.y;
        wl[4 * c + 2] = u0.z ^ m0.z; wl[4 * c + 3] = u0.w ^ m0.w;
        wh[4 * c + 0] = u1.x ^ m1.x; wh[4 * c + 1] = u1.y ^ m1.y;
        wh[4 * c + 2] = u1.z ^ m1.z; wh[4 * c + 3] = u1.w ^ m1.w;
      }
      uint64_t acc = pk2(0.f, 0.f);
#pragma unroll
      for (int q = 0; q < 32; ++q) {
        // elements 2q, 2q + 1 and 64 + 2q, 64 + 2q + 1
        const float a0 = __uint_as_float(wl[q] << 16), a1 = __uint_as_float(wl[q] & 0xffff0000u);
        const float b0 = __uint_as_float(wh[q] << 16), b1 = __uint_as_float(wh[q] & 0xffff0000u);
        const uint64_t e0 = pk2(a0, b0), e1 = pk2(a1, b1);
        acc = fma2(e0, e0, acc);
        acc = fma2(e1, e1, acc);
        // first butterfly stage (distance 64): (x_p + x_{p+64}, x_p - x_{p+64})
        P[2 * q] = pk2(a0 + b0, a0 - b0);
        P[2 * q + 1] = pk2(a1 + b1, a1 - b1);
      }
      const float2 s2 = up2(acc);
      ss = s2.x + s2.y;
    }
    // ---- remaining butterfly stages on pair indices (distances 1 .. 32)
#pragma unroll
    for (int h = 1; h < 64; h <<= 1) {
#pragma unroll
      for (int p = 0; p < 64; ++p) {
        if ((p & h) == 0) {
          const uint64_t u = P[p], v = P[p + h];
          P[p] = add2(u, v);
          P[p + h] = sub2(u, v);
        }
      }
    }
    const float n = sqrtf(ss);
    const __half n16 = __float2half_rn(n);
    const float n16f = __half2float(n16);

    // ---- previous tile: wait for its MMA, take the sign bits of D
    if (k > 0) {
      if (!__syncthreads_and(mbar_wait_ns(&bar_mma, static_cast<uint32_t>((k - 1) & 1), kWaitNs))) {
        failed = true;
        break;
      }
      tc_fence_after();
      store_signs(a, tlane, prev_valid, prev_row);
    }

    // ---- decisions, packed indices, residual, fp16 hi/lo halves into tensor memory
    float T[NL - 1];
#pragma unroll
    for (int t = 0; t < NL - 1; ++t) T[t] = n > 0.f ? thr[t] * n : thr[t];
    // power-of-two scale keeping |rho| * scl below 2^15 (|rho_j| <= (sqrt(d) + 2.2) n)
    const uint32_t ex = (__float_as_uint(n) >> 23) & 0xffu;
    const float scl = __uint_as_float((ex >= 10u ? 264u - ex : 254u) << 23);
    const uint64_t scl2 = pk2(scl, scl);
    const uint64_t mn2 = pk2(-n16f, -n16f);
    uint32_t pk[NW];
#pragma unroll
    for (int w = 0; w < NW; ++w) pk[w] = 0u;
    uint64_t racc = pk2(0.f, 0.f);
#pragma unroll
    for (int g = 0; g < 8; ++g) {
      uint32_t hw[8], lw[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int p = 8 * g + i;
        const float2 y = up2(P[p]);
        float c2[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float yv = e ? y.y : y.x;
          const int j = p + 64 * e;
          uint32_t id = 0;
          float c = cen[0];
#pragma unroll
          for (int t = 0; t < NL - 1; ++t) {
            const bool gt = yv > T[t];
            id += gt ? 1u : 0u;
            c = gt ? cen[t + 1] : c;
          }
          pk[(j * W) >> 5] |= id << ((j * W) & 31);
          c2[e] = c;
        }
        const uint64_t r = fma2(mn2, pk2(c2[0], c2[1]), P[p]);
        racc = fma2(r, r, racc);
        const float2 v = up2(mul2(r, scl2));
        const uint32_t hb = h2_bits(v.x, v.y);
        const float2 hf = __half22float2(*reinterpret_cast<const __half2*>(&hb));
        const float2 lo = up2(sub2(pk2(v.x, v.y), pk2(hf.x, hf.y)));
        hw[i] = hb;
        lw[i] = h2_bits(lo.x, lo.y);
      }
      tmem_st8(tlane + 128 + 8 * g, hw);
      tmem_st8(tlane + 192 + 8 * g, lw);
    }
    const float2 r2 = up2(racc);
    const __half r16 = __float2half_rn(sqrtf((r2.x + r2.y) * (1.f / 128.f)));
    if (valid) {
      const int64_t orow = out_row_tc(a.map, row);
      uint4* dst = reinterpret_cast<uint4*>(a.idx + orow * IB);
#pragma unroll
      for (int w = 0; w < NW; w += 4) dst[w / 4] = make_uint4(pk[w], pk[w + 1], pk[w + 2], pk[w + 3]);
      *reinterpret_cast<uint32_t*>(a.nrm + orow * 2) =
          static_cast<uint32_t>(half_bits(n16)) | (static_cast<uint32_t>(half_bits(r16)) << 16);
    }
    prev_row = row;
    prev_valid = valid;

    // ---- issue the MMAs of this tile; refill this staging buffer two tiles ahead
    tmem_st_wait();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int s = 0; s < 16; ++s) {
        const uint64_t bdesc = umma_desc(smem_u32(sB) + (s & 7) * 256, 128, 2048);
        umma_f16_ts(tbase, tbase + 128 + 8 * s, bdesc, idesc, s > 0 ? 1u : 0u);
      }
      umma_commit(&bar_mma);
    }
    if (warp == 0 && k + 2 < n_local) issue_tile(a, sX + b * kXBuf, &bar_x[b], tile + 2 * grid, lane);
  }

  if (!failed && n_local > 0) {
    // sign bits of the last tile
    if (__syncthreads_and(mbar_wait_ns(&bar_mma, static_cast<uint32_t>((n_local - 1) & 1), kWaitNs))) {
      tc_fence_after();
      store_signs(a, tlane, prev_valid, prev_row);
    } else {
      failed = true;
    }
  }
  if (failed) {
    // a bounded wait gave up: report, let outstanding copies and MMAs land (bounded), leave
    if (tid == 0) atomicOr(a.err, 1);
    for (int bb = 0; bb < 2; ++bb) mbar_wait_ns(&bar_x[bb], 0, kWaitNs / 4);
    mbar_wait_ns(&bar_mma, 0, kWaitNs / 4);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, kTmemCols);
  }
}

template <int MB>
tq_status run_tc(const TcKeyArgs& a, cudaStream_t st) {
  auto kern = k_keys_prod_tc<MB>;
  static bool attr_set = false;
  if (!attr_set) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) !=
        cudaSuccess)
      return TQ_ECUDA;
    attr_set = true;
  }
  int dev = 0;
  cudaGetDevice(&dev);
  const int64_t cap = 2ll * sm_count(dev);
  const int grid = static_cast<int>(a.n_tiles < cap ? a.n_tiles : cap);
  kern<<<grid, 128, kSmemBytes, st>>>(a);
  return cudaGetLastError() == cudaSuccess ? TQ_OK : TQ_ECUDA;
}

}  // namespace

__device__ int g_tq_device_error = 0;

bool keys_tc_ok(const tq_quantizer* q, int dtype) {
  return q->mode == TQ_MODE_PROD && dtype == TQ_BF16 && q->bits >= 2 && q->bits <= 4;
}

tq_status launch_keys_tc(const tq_quantizer* q, const void* x, int64_t n_rows, int64_t ld,
                         tq_key_planes out, RowMap map, cudaStream_t st) {
  if (n_rows == 0) return TQ_OK;
  int* err = nullptr;
  if (cudaGetSymbolAddress(reinterpret_cast<void**>(&err), g_tq_device_error) != cudaSuccess)
    return TQ_ECUDA;
  TcKeyArgs a{static_cast<const uint16_t*>(x), n_rows, ld, (n_rows + kTile - 1) / kTile,
              q->dev, out.idx, out.signs, out.norms, map, err};
  switch (q->bits) {
    case 2: return run_tc<1>(a, st);
    case 3: return run_tc<2>(a, st);
    case 4: return run_tc<3>(a, st);
    default: return TQ_EUNSUPPORTED;
  }
}

tq_status take_device_error(cudaStream_t st) {
  if (cudaStreamSynchronize(st) != cudaSuccess) return TQ_ECUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_tq_device_error, sizeof(int)) != cudaSuccess) return TQ_ECUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_tq_device_error, &zero, sizeof(int)) != cudaSuccess) return TQ_ECUDA;
    return TQ_ETIMEOUT;
  }
  return TQ_OK;
}

}  // namespace tq
