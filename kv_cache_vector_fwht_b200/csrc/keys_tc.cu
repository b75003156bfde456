// prod-mode key quantization of bf16 rows with the QJL projection on the 5th-generation
// tensor cores (sm_100a: TMA, tcgen05.mma, tensor memory).
//
// What is computed (tqlite README: rotation.py, codebook.py, prod.py; Implementing TurboQuant
// (part 5), algorithm overview; TurboQuant bit-packing article sections 2-4), per row x:
//   n = ||x||, y = H (s . x) (unnormalised Sylvester Hadamard, so Pi x = y / sqrt(d)),
//   idx_j = #{k : y_j > t_k n}, rho = y - n16 C[idx] (= sqrt(d) Pi r), ||r|| = ||rho|| / sqrt(d),
//   QJL bits [(S_rot rho)_j >= 0] (= [(S r)_j >= 0] with S = S_rot Pi).
//
// Work split. A CTA of four warps owns a tile of 128 rows: thread i owns row i of the tile,
// which is also lane i of its tensor-memory (TMEM) region. Per tile:
//   1. TMA brings the 128 x 256 B tile into shared memory (two 64-column boxes, 128-byte
//      swizzle, double-buffered one tile ahead).
//   2. Each thread reads its row, applies the rotation signs, takes the norm and runs all
//      seven butterfly stages of the Hadamard transform in registers.
//   3. It takes the sign bits of the previous tile's QJL product from the accumulator
//      columns, then parks its transformed row in those same columns.
//   4. A rolled loop over column groups reloads the row from TMEM, makes the codebook
//      decisions, packs the indices and writes the residual -- scaled by a power of two and
//      split into fp16 hi + lo halves -- into TMEM as the MMA's A operand (128 x 256, K = hi
//      then lo).
//   5. When all 128 threads have arrived on an mbarrier, one thread issues sixteen m128 n128
//      k16 tcgen05.mma with S_rot (fp16-exact, shared memory, B operand) and commits them to
//      a second mbarrier: D = [hi | lo] [S | S]^T in fp32. The products of fp16 values are
//      exact in fp32, so D carries the fp32 accuracy of S_rot rho.
// No CTA-wide barrier sits inside the tile loop; every wait is an mbarrier wait bounded in
// time, after which the kernel records an error (tq_sync_status) and skips further work.
//
// Registers hold the row as 64 fp32 pairs (y_p, y_{p + 64}); the K order of both MMA
// operands is permuted to match (k' = 2p holds element p, k' = 2p + 1 element p + 64), which
// leaves the product unchanged.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "tq_device.cuh"
#include "tq_internal.h"

namespace tq {
namespace {

constexpr int kTile = 128;             // rows per tile = MMA M = TMEM lanes
constexpr int kXBuf = kTile * 256;     // one staged tile (two 16 KB swizzled boxes)
constexpr int kBBytes = kD * kD * 2;   // S_rot operand
constexpr int kMaskOff = kBBytes + 2 * kXBuf;
constexpr int kCodeOff = kMaskOff + 256;
constexpr int kSmemBytes = kCodeOff + 16 * kTile * 4;
constexpr uint32_t kTmemCols = 256;    // D: columns [0, 128); A: hi [128, 192), lo [192, 256)
constexpr uint64_t kWaitNs = 2000000000ull;
constexpr int64_t kChunkRows = int64_t(1) << 30;  // rows per launch (TMA row coordinate is int32)

struct TcKeyArgs {
  int64_t n_rows;    // rows of this launch
  int64_t row_base;  // global index of its first row
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

// 1.0f if a > b else 0.0f (an exact compare)
// m + 1/2 with m = #{k < 7 : a > T[OFF + k]} for ascending T[OFF .. OFF + 6] (the positive
// thresholds of a 16-level codebook), by binary search: the same strict compares as the
// ladder over all seven, along one path of three, so the count is identical.
template <int OFF, int N>
__device__ __forceinline__ float mag_half7(float a, const float (&T)[N]) {
  static_assert(OFF + 7 <= N, "seven thresholds");
  const bool b4 = a > T[OFF + 3];
  const bool b2 = a > (b4 ? T[OFF + 5] : T[OFF + 1]);
  const float t1 = b4 ? (b2 ? T[OFF + 6] : T[OFF + 4]) : (b2 ? T[OFF + 2] : T[OFF + 0]);
  const bool b1 = a > t1;
  return (b4 ? 4.f : 0.f) + (b2 ? 2.f : 0.f) + (b1 ? 1.5f : 0.5f);
}

__device__ __forceinline__ float gt_one(float a, float b) {
  float d;
  asm("set.gt.f32.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
  return d;
}

// Bits [d_i >= 0] of 32 fp32 values taken from their sign bits (a -0 result cannot occur for
// a nonzero residual; all-zero residual rows are handled by the caller). Byte permutes gather
// the top bytes of d[m], d[m+8], d[m+16], d[m+24] into one word whose sign bits are then
// shifted into bit positions m, m + 8, m + 16, m + 24.
__device__ __forceinline__ uint32_t sign_word(const uint32_t (&d)[32]) {
  uint32_t acc = 0;
#pragma unroll
  for (int m = 0; m < 8; ++m) {
    const uint32_t t1 = __byte_perm(d[m], d[m + 8], 0x0073);
    const uint32_t t2 = __byte_perm(d[m + 16], d[m + 24], 0x0073);
    const uint32_t g = __byte_perm(t1, t2, 0x5410);
    const uint32_t sh = m < 7 ? __umulhi(g, 1u << (25 + m)) : g;  // g >> (7 - m)
    acc |= sh & (0x01010101u << m);
  }
  return ~acc;
}

// Sign bits of this thread's accumulator row (its TMEM lane), stored as the row's 16-byte
// sign plane.
__device__ __forceinline__ void store_signs(const TcKeyArgs& a, uint32_t tlane, bool valid,
                                            bool zero_res, int64_t grow) {
  uint32_t sg[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t d[32];
    tmem_ld32_sync(tlane + 32 * q, d);
    sg[q] = sign_word(d);
  }
  if (zero_res) sg[0] = sg[1] = sg[2] = sg[3] = 0xffffffffu;  // S_rot 0 = 0 >= 0
  if (valid)
    *reinterpret_cast<uint4*>(a.sgn + out_row_tc(a.map, grow) * 16) =
        make_uint4(sg[0], sg[1], sg[2], sg[3]);
}

// PROD: prod keys (MB = bits - 1, residual + QJL on tcgen05); else mse keys (MB = bits,
// indices and the norm only; the accumulator columns only park the rotated row).
template <bool PROD, int MB>
__global__ void __launch_bounds__(128, 2)
    k_keys_tc(const __grid_constant__ CUtensorMap tmap, const __grid_constant__ TcKeyArgs a) {
  constexpr int NL = 1 << MB;
  constexpr uint32_t TCOLS = PROD ? kTmemCols : 128u;
  constexpr int W = storage_width_c(MB);
  constexpr int NW = 4 * W;       // index words per row
  constexpr int GP = 32 / W;      // pairs per decision group: one index word per half
  constexpr int NG = 64 / GP;     // decision groups

  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* sB = smem;
  uint8_t* sX = smem + kBBytes;
  const uint32_t* sMask = reinterpret_cast<const uint32_t*>(smem + kMaskOff);
  uint32_t* sCode = reinterpret_cast<uint32_t*>(smem + kCodeOff);
  __shared__ __align__(8) uint64_t bar_x[2];
  __shared__ __align__(8) uint64_t bar_b;
  __shared__ __align__(8) uint64_t bar_mma;
  __shared__ __align__(8) uint64_t bar_a;
  __shared__ uint32_t tslot;

  const int tid = threadIdx.x, warp = tid >> 5;
  const DevTables* __restrict__ tab = a.tab;
  const int64_t grid = gridDim.x;
  const int64_t n_local = (a.n_tiles - blockIdx.x + grid - 1) / grid;  // grid <= n_tiles

  if (warp == 0) {
    tmem_alloc(&tslot, TCOLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&bar_x[0], 1);
    mbar_init(&bar_x[1], 1);
    mbar_init(&bar_b, 1);
    mbar_init(&bar_mma, 1);
    mbar_init(&bar_a, kTile);
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = tslot;
  const uint32_t tlane = tbase + (static_cast<uint32_t>(warp * 32) << 16);

  if (tid == 0) {
    mbar_expect_tx(&bar_b, (PROD ? kBBytes : 0) + 256);
    if constexpr (PROD) bulk_g2s(sB, tab->s_umma, kBBytes, &bar_b);
    bulk_g2s(smem + kMaskOff, tab->pair_mask, 256, &bar_b);
    for (int k = 0; k < 2 && k < n_local; ++k) {
      const int row0 = static_cast<int>((blockIdx.x + k * grid) * kTile);
      mbar_expect_tx(&bar_x[k], kXBuf);
      tma_load_2d(sX + k * kXBuf, &tmap, 0, row0, &bar_x[k]);
      tma_load_2d(sX + k * kXBuf + kXBuf / 2, &tmap, 64, row0, &bar_x[k]);
    }
  }

  float thr[NL - 1], cen[NL];
#pragma unroll
  for (int k = 0; k < NL - 1; ++k) thr[k] = tab->thr[0][k];
#pragma unroll
  for (int k = 0; k < NL; ++k) cen[k] = tab->cent[0][k];

  constexpr uint32_t idesc = umma_idesc_f16(kTile, kD);
  bool ok = mbar_wait_ns(&bar_b, 0, kWaitNs);
  int64_t prev_row = 0;
  bool prev_valid = false, prev_zero = false;
  const uint32_t sw = static_cast<uint32_t>(tid & 7);  // 128-byte swizzle phase of this row

  for (int64_t k = 0; k < n_local; ++k) {
    const int b = static_cast<int>(k & 1);
    const int64_t tile = blockIdx.x + k * grid;
    const int64_t row = tile * kTile + tid;
    const bool valid = row < a.n_rows;
    if (ok) ok = mbar_wait_ns(&bar_x[b], static_cast<uint32_t>((k >> 1) & 1), kWaitNs);

    // ---- row from shared memory: signs, first butterfly stage, norm.
    // P[p] = (x_p + x_{p+64}, x_p - x_{p+64}) after the distance-64 stage.
    uint64_t P[64];
    uint64_t nacc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) nacc[i] = pk2(0.f, 0.f);
    {
      const uint8_t* x0 = sX + b * kXBuf + tid * 128;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint32_t off = (static_cast<uint32_t>(c) ^ sw) << 4;
        const uint4 u0 = *reinterpret_cast<const uint4*>(x0 + off);
        const uint4 u1 = *reinterpret_cast<const uint4*>(x0 + kXBuf / 2 + off);
        const uint4 m0 = *reinterpret_cast<const uint4*>(sMask + 4 * c);
        const uint4 m1 = *reinterpret_cast<const uint4*>(sMask + 32 + 4 * c);
        const uint32_t wl[4] = {u0.x ^ m0.x, u0.y ^ m0.y, u0.z ^ m0.z, u0.w ^ m0.w};
        const uint32_t wh[4] = {u1.x ^ m1.x, u1.y ^ m1.y, u1.z ^ m1.z, u1.w ^ m1.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float a0 = __uint_as_float(wl[i] * 65536u), a1 = __uint_as_float(wl[i] & 0xffff0000u);
          const float b0 = __uint_as_float(wh[i] * 65536u), b1 = __uint_as_float(wh[i] & 0xffff0000u);
          const int p = 8 * c + 2 * i;
          P[p] = pk2(a0 + b0, a0 - b0);
          P[p + 1] = pk2(a1 + b1, a1 - b1);
          nacc[(2 * i) & 7] = fma2(P[p], P[p], nacc[(2 * i) & 7]);
          nacc[(2 * i + 1) & 7] = fma2(P[p + 1], P[p + 1], nacc[(2 * i + 1) & 7]);
        }
      }
    }
    // ---- butterfly stages of distance 1 .. 32 on pair indices
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
    // (a + b)^2 + (a - b)^2 = 2 (a^2 + b^2)
#pragma unroll
    for (int i = 1; i < 8; i <<= 1)
#pragma unroll
      for (int j = 0; j < 8; j += 2 * i) nacc[j] = add2(nacc[j], nacc[j + i]);
    const float2 n2 = up2(nacc[0]);
    const float n = sqrtf((n2.x + n2.y) * 0.5f);
    const __half n16 = __float2half_rn(n);
    const float n16f = __half2float(n16);

    // ---- previous tile: sign bits of its QJL product
    if (PROD && k > 0) {
      if (ok) ok = mbar_wait_ns(&bar_mma, static_cast<uint32_t>((k - 1) & 1), kWaitNs);
      tc_fence_after();
      store_signs(a, tlane, prev_valid, prev_zero, a.row_base + prev_row);
    }

    // ---- park the transformed row in the accumulator columns (pair p -> columns 2p, 2p + 1)
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      uint32_t r[16];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float2 v = up2(P[8 * q + i]);
        r[2 * i] = __float_as_uint(v.x);
        r[2 * i + 1] = __float_as_uint(v.y);
      }
      tmem_st16(tlane + 16 * q, r);
    }
    tmem_st_wait();

    // ---- per-row decision tables. Power-of-two scale scl keeps |rho| scl below 2^15
    // (|rho_j| <= (sqrt(d) + 2.2) n); ncs[k] = -scl RN(n16 C_k), so rho scl = fma(y, scl, ncs).
    float T[NL - 1];
#pragma unroll
    for (int t = 0; t < NL - 1; ++t) T[t] = n > 0.f ? thr[t] * n : thr[t];
    const uint32_t ex = (__float_as_uint(n) >> 23) & 0xffu;
    const float scl = PROD ? __uint_as_float((ex >= 10u ? 264u - ex : 254u) << 23) : 1.f;
    // The centroid term of code c is ncs[0] + sum_{t < c} dcs[t]: a multiply-add per exact
    // 0/1 compare (its rounding moves rho by about an ulp, far inside the parity margins).
    float ncs[NL];
#pragma unroll
    for (int t = 0; t < NL; ++t) ncs[t] = -(n16f * cen[t]) * scl;
    uint64_t dcs2[NL - 1], T2[NL - 1];
#pragma unroll
    for (int t = 0; t < NL - 1; ++t) {
      dcs2[t] = pk2(ncs[t + 1] - ncs[t], ncs[t + 1] - ncs[t]);
      T2[t] = pk2(T[t], T[t]);
    }
    const uint64_t ncs02 = pk2(ncs[0], ncs[0]);
    const uint64_t scl2 = pk2(scl, scl);
    // Symmetric codebooks (C_{L-1-k} = -C_k, t_{L-2-k} = -t_k, middle threshold 0), used for
    // L >= 8: with s = [y > 0], sigma = 2 s - 1 and m = #{t < H : |y| > T+_t} over the
    // H = L/2 - 1 positive thresholds, code = (L - 1)/2 + sigma (m + 1/2) and the centroid is
    // sigma C+_m. (|y| on a positive threshold, a tie, may take the neighbouring code.)
    constexpr bool SYM = NL >= 8;
    constexpr int H = NL / 2 - 1;
    float TP[SYM ? H : 1];
    uint64_t dcsP2[SYM ? H : 1];
#pragma unroll
    for (int t = 0; t < H; ++t) {
      TP[t] = T[NL / 2 + t];
      dcsP2[t] = pk2(ncs[NL / 2 + t + 1] - ncs[NL / 2 + t], ncs[NL / 2 + t + 1] - ncs[NL / 2 + t]);
    }
    const uint64_t ncsP02 = pk2(ncs[NL / 2], ncs[NL / 2]);

    uint64_t racc[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) racc[i] = pk2(0.f, 0.f);
    // decisions of column group g (pairs [GP g, GP g + GP)) from its TMEM columns yg
    auto decide_group = [&](int g, const uint32_t (&yg)[GP / 8][16]) {
      // index words of elements [GP g, GP g + GP) (.x) and +64 (.y), accumulated in fp32 as
      // exact integers: codes of pairs [0, GP/2) in wa, [GP/2, GP) in wb (each < 2^16)
      // symmetric path: each word starts at sum_j kw_j (L - 1)/2 over its pairs
      constexpr float kW0 = SYM ? 0.5f * (NL - 1) * (W == 4 ? 4369.f : W == 2 ? 21845.f : 65535.f) : 0.f;
      uint64_t wa = pk2(kW0, kW0), wb = pk2(kW0, kW0);
      uint32_t hw[GP], lw[GP];
#pragma unroll
      for (int q = 0; q < GP / 8; ++q) {
        const uint32_t (&yv)[16] = yg[q];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int pi = 8 * q + i;  // pair index within the group
          // index = number of thresholds below y: each exact 0/1 compare adds 2^(W slot) to
          // the word and one centroid step to the residual's offset
          const float kw = static_cast<float>(1u << (W * (pi % (GP / 2))));
          const uint64_t kw2 = pk2(kw, kw);
          const uint64_t y2 = pk2(__uint_as_float(yv[2 * i]), __uint_as_float(yv[2 * i + 1]));
          uint64_t c2 = SYM ? ncsP02 : ncs02;
          uint64_t sg2 = 0ull;
          if constexpr (SYM) {
            const float y0 = __uint_as_float(yv[2 * i]), y1 = __uint_as_float(yv[2 * i + 1]);
            const uint64_t s2 = pk2(gt_one(y0, 0.f), gt_one(y1, 0.f));
            const uint64_t sk2 = fma2(s2, pk2(2.f * kw, 2.f * kw), pk2(-kw, -kw));  // sigma kw
            uint64_t w = pi < GP / 2 ? wa : wb;
            const float a0 = fabsf(y0), a1 = fabsf(y1);
            if constexpr (H == 7 && !PROD) {
              // 16 levels: m + 1/2 by binary search over the positive thresholds
              w = fma2(sk2, pk2(mag_half7<0>(a0, TP), mag_half7<0>(a1, TP)), w);
            } else {
              w = fma2(sk2, pk2(0.5f, 0.5f), w);
#pragma unroll
              for (int t = 0; t < H; ++t) {
                const uint64_t ind = pk2(gt_one(a0, TP[t]), gt_one(a1, TP[t]));
                if constexpr (PROD) c2 = fma2(ind, dcsP2[t], c2);
                w = fma2(ind, sk2, w);
              }
            }
            if (pi < GP / 2) wa = w;
            else wb = w;
            if constexpr (PROD) sg2 = fma2(s2, pk2(2.f, 2.f), pk2(-1.f, -1.f));
          } else {
#pragma unroll
            for (int t = 0; t < NL - 1; ++t) {
              const float2 th = up2(T2[t]);
              const uint64_t ind = pk2(gt_one(__uint_as_float(yv[2 * i]), th.x),
                                       gt_one(__uint_as_float(yv[2 * i + 1]), th.y));
              if constexpr (PROD) c2 = fma2(ind, dcs2[t], c2);
              if (pi < GP / 2) wa = fma2(ind, kw2, wa);
              else wb = fma2(ind, kw2, wb);
            }
          }
          if constexpr (!PROD) continue;
          const uint64_t r = SYM ? fma2(sg2, c2, mul2(y2, scl2)) : fma2(y2, scl2, c2);
          racc[pi & 3] = fma2(r, r, racc[pi & 3]);
          // hi/lo split: hi = r with its 13 low mantissa bits cleared (11 significant bits,
          // exact in fp16 for |r| < 2^15), lo = r - hi exactly in fp32 (at most 13 significant
          // bits, rounded to fp16's 11): |r - hi16 - lo16| <= 2^-21 |r|
          const float2 rv = up2(r);
          const float hx = __uint_as_float(__float_as_uint(rv.x) & 0xffffe000u);
          const float hy = __uint_as_float(__float_as_uint(rv.y) & 0xffffe000u);
          const float2 lv = up2(sub2(r, pk2(hx, hy)));
          hw[pi] = h2_bits(hx, hy);
          lw[pi] = h2_bits(lv.x, lv.y);
        }
      }
      if constexpr (!PROD) {
      } else if constexpr (GP == 8) {
        tmem_st8(tlane + 128 + GP * g, *reinterpret_cast<uint32_t(*)[8]>(hw));
        tmem_st8(tlane + 192 + GP * g, *reinterpret_cast<uint32_t(*)[8]>(lw));
      } else {
#pragma unroll
        for (int q = 0; q < GP / 16; ++q) {
          tmem_st16(tlane + 128 + GP * g + 16 * q, *reinterpret_cast<uint32_t(*)[16]>(hw + 16 * q));
          tmem_st16(tlane + 192 + GP * g + 16 * q, *reinterpret_cast<uint32_t(*)[16]>(lw + 16 * q));
        }
      }
      {
        // exact integers below 2^16: adding 2^23 puts them in the low mantissa bits
        const float2 fa = up2(add2(wa, pk2(8388608.f, 8388608.f)));
        const float2 fb = up2(add2(wb, pk2(8388608.f, 8388608.f)));
        constexpr int kHalfBits = W * GP / 2;
        sCode[g * kTile + tid] = (__float_as_uint(fa.x) & 0xffffu) |
                                 ((__float_as_uint(fb.x) & 0xffffu) << kHalfBits);
        sCode[(NG + g) * kTile + tid] = (__float_as_uint(fa.y) & 0xffffu) |
                                        ((__float_as_uint(fb.y) & 0xffffu) << kHalfBits);
      }
    };
    // The loads of group g + 1 are issued before group g's decisions and waited for after
    // them, so the TMEM latency overlaps the work (NG is even).
    auto issue = [&](int g, uint32_t (&yg)[GP / 8][16]) {
#pragma unroll
      for (int q = 0; q < GP / 8; ++q) tmem_ld16(tlane + 2 * GP * g + 16 * q, yg[q]);
    };
    auto tie = [&](uint32_t (&yg)[GP / 8][16]) {
#pragma unroll
      for (int q = 0; q < GP / 8; ++q) tmem_ld_wait_tied16(yg[q]);
    };
    // (prod with 1- or 2-bit indices keeps one group in flight: a second buffer would spill)
    constexpr bool kAhead = !(PROD && MB <= 2);
    static_assert(NG % 2 == 0, "column groups come in pairs");
    uint32_t yA[GP / 8][16];
    if constexpr (kAhead) {
      uint32_t yB[GP / 8][16];
      issue(0, yA);
      tie(yA);
#pragma unroll 1
      for (int g = 0; g < NG; g += 2) {
        issue(g + 1, yB);
        decide_group(g, yA);
        tie(yB);
        if (g + 2 < NG) issue(g + 2, yA);
        decide_group(g + 1, yB);
        if (g + 2 < NG) tie(yA);
      }
    } else {
#pragma unroll 1
      for (int g = 0; g < NG; ++g) {
        issue(g, yA);
        tie(yA);
        decide_group(g, yA);
      }
    }
    const float2 r2 = up2(add2(add2(racc[0], racc[1]), add2(racc[2], racc[3])));
    const float rss = r2.x + r2.y;
    const __half r16 = __float2half_rn(sqrtf(rss * (1.f / 128.f)) / scl);
    if (valid) {
      const int64_t orow = out_row_tc(a.map, a.row_base + row);
      uint4* dst = reinterpret_cast<uint4*>(a.idx + orow * (NW * 4));
#pragma unroll
      for (int w = 0; w < NW; w += 4)
        dst[w / 4] = make_uint4(sCode[w * kTile + tid], sCode[(w + 1) * kTile + tid],
                                sCode[(w + 2) * kTile + tid], sCode[(w + 3) * kTile + tid]);
      if constexpr (PROD)
        *reinterpret_cast<uint32_t*>(a.nrm + orow * 2) =
            static_cast<uint32_t>(half_bits(n16)) | (static_cast<uint32_t>(half_bits(r16)) << 16);
      else
        a.nrm[orow] = half_bits(n16);
    }
    prev_row = row;
    prev_valid = valid;
    prev_zero = !(rss > 0.f);

    // ---- hand the tile to the tensor core; refill this staging buffer two tiles ahead
    tmem_st_wait();
    tc_fence_before();
    mbar_arrive(&bar_a);
    if (tid == 0) {
      if (ok) ok = mbar_wait_ns(&bar_a, static_cast<uint32_t>(k & 1), kWaitNs);
      tc_fence_after();
      if (ok) {
        if constexpr (PROD) {
#pragma unroll
          for (int s = 0; s < 16; ++s) {
            const uint64_t bdesc = umma_desc(smem_u32(sB) + (s & 7) * 256, 128, 2048);
            umma_f16_ts(tbase, tbase + 128 + 8 * s, bdesc, idesc, s > 0 ? 1u : 0u);
          }
          umma_commit(&bar_mma);
        }
        if (k + 2 < n_local) {
          const int row0 = static_cast<int>((tile + 2 * grid) * kTile);
          mbar_expect_tx(&bar_x[b], kXBuf);
          tma_load_2d(sX + b * kXBuf, &tmap, 0, row0, &bar_x[b]);
          tma_load_2d(sX + b * kXBuf + kXBuf / 2, &tmap, 64, row0, &bar_x[b]);
        }
      }
    }
  }

  if (PROD && n_local > 0) {
    if (ok) ok = mbar_wait_ns(&bar_mma, static_cast<uint32_t>((n_local - 1) & 1), kWaitNs);
    tc_fence_after();
    if (ok) store_signs(a, tlane, prev_valid, prev_zero, a.row_base + prev_row);
  }
  if (!ok) atomicOr(a.err, 1);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, TCOLS);
  }
}

// ---------------------------------------------------------------------------------------
// Grouped keys (tqlite grouped.py; TurboQuant overview, "three quantization modes" table):
// the 32 outlier channels form a group quantized at b + 1 bits and the other 96 a group at
// b bits. Each group has its own norm and is rotated by 32-point Hadamard blocks after its
// own signs; in chain order (outlier channels ascending, then normal channels ascending)
// block k holds chain positions 32k .. 32k + 31, and u_j > t_k / sqrt(d_g) is decided as
// y_j > t_k ||x_g|| sqrt(32 / d_g) on the unnormalised block transform y.
//
// Same tiling as k_keys_tc (128-row TMA tiles, one thread per row, the transformed row parked
// in TMEM for a rolled decision loop), with a gather in front: once a tile has landed, each
// warp copies its 32 rows into chain order in a padded shared-memory buffer (lane l moves
// the natural channels 4l .. 4l + 3 of a row), which also releases the TMA buffer. The four
// transforms run on fp32 pairs (y_p, y_{p+64}): blocks 0 and 2 share pair indices 0..31,
// blocks 1 and 3 pair indices 32..63, so every butterfly is one packed add or subtract.
// ---------------------------------------------------------------------------------------
constexpr int kGStride = 272;                    // bytes per chain-ordered row (256 + 16)
constexpr int kGPermOff = 2 * kXBuf;
constexpr int kGMaskOff = kGPermOff + kTile * kGStride;
constexpr int kGPosOff = kGMaskOff + 256;        // chain position of each channel (uint16)
constexpr int kGCodeOff = kGPosOff + 256;        // packed halfwords [32][kTile] (uint16)
constexpr int kGSmemBytes = kGCodeOff + 32 * kTile * 2;

// Codes of 16 values (pairs i, i + 8 of yv) against NT ascending thresholds, packed
// LSB-first at width W into W halfwords sCode[(hw0 + j) kTile + tid], j < W. Exact 0/1
// compares are summed with power-of-two weights as exact fp32 integers below 2^16.
template <int W, int NT>
__device__ __forceinline__ void decide16(const uint32_t (&yv)[16], const float (&T)[NT],
                                         uint16_t* sCode, int hw0, int tid) {
  constexpr int NA = W == 4 ? 2 : 1;
  // L = NT + 1 >= 8 (4-bit fields): symmetric codebook, code = (L - 1)/2 + sigma (m + 1/2)
  // with m counted on |y| against the H positive thresholds (as in k_keys_tc)
  constexpr bool SYM = NT >= 7;
  constexpr int H = (NT + 1) / 2 - 1;
  uint64_t acc[NA];
#pragma unroll
  for (int j = 0; j < NA; ++j) acc[j] = SYM ? pk2(0.5f * NT * 4369.f, 0.5f * NT * 4369.f) : pk2(0.f, 0.f);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int slot = W == 4 ? 4 * (i & 3) : W * i;
    const float wx = static_cast<float>(1u << slot);
    const float wy = W == 1 ? static_cast<float>(1u << (i + 8)) : wx;
    const uint64_t kw = pk2(wx, wy);
    const float y0 = __uint_as_float(yv[i]), y1 = __uint_as_float(yv[i + 8]);
    uint64_t& A = acc[W == 4 ? i / 4 : 0];
    if constexpr (SYM) {
      const uint64_t s2 = pk2(gt_one(y0, 0.f), gt_one(y1, 0.f));
      const uint64_t sk2 = fma2(s2, pk2(2.f * wx, 2.f * wx), pk2(-wx, -wx));  // sigma kw
      const float a0 = fabsf(y0), a1 = fabsf(y1);
      if constexpr (H == 7) {
        // 16 levels: m + 1/2 by binary search over the positive thresholds
        A = fma2(sk2, pk2(mag_half7<H + 1>(a0, T), mag_half7<H + 1>(a1, T)), A);
      } else {
        A = fma2(sk2, pk2(0.5f, 0.5f), A);
#pragma unroll
        for (int t = 0; t < H; ++t) A = fma2(pk2(gt_one(a0, T[H + 1 + t]), gt_one(a1, T[H + 1 + t])), sk2, A);
      }
    } else {
#pragma unroll
      for (int t = 0; t < NT; ++t) A = fma2(pk2(gt_one(y0, T[t]), gt_one(y1, T[t])), kw, A);
    }
  }
  auto bits16 = [](float f) {  // an exact integer below 2^16 lands in the low mantissa bits
    return static_cast<uint16_t>(__float_as_uint(f + 8388608.f) & 0xffffu);
  };
  if constexpr (W == 1) {
    const float2 v = up2(acc[0]);
    sCode[hw0 * kTile + tid] = bits16(v.x + v.y);
  } else if constexpr (W == 2) {
    const float2 v = up2(acc[0]);
    sCode[hw0 * kTile + tid] = bits16(v.x);
    sCode[(hw0 + 1) * kTile + tid] = bits16(v.y);
  } else {
    const float2 v0 = up2(acc[0]), v1 = up2(acc[1]);
    sCode[hw0 * kTile + tid] = bits16(v0.x);
    sCode[(hw0 + 1) * kTile + tid] = bits16(v1.x);
    sCode[(hw0 + 2) * kTile + tid] = bits16(v0.y);
    sCode[(hw0 + 3) * kTile + tid] = bits16(v1.y);
  }
}

template <int B>
__global__ void __launch_bounds__(128, 2)
    k_keys_grp_tc(const __grid_constant__ CUtensorMap tmap, const __grid_constant__ TcKeyArgs a) {
  constexpr int NTO = (1 << (B + 1)) - 1, NTN = (1 << B) - 1;
  constexpr int WO = storage_width_c(B + 1), WN = storage_width_c(B);
  constexpr int HWO = 2 * WO;           // halfwords of the outlier group (32 codes)
  constexpr int NHW = HWO + 6 * WN;     // halfwords per row
  constexpr int IB = 2 * NHW;           // index bytes per row: 20, 40, 64

  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* sX = smem;
  uint8_t* sP = smem + kGPermOff;
  const uint32_t* sMask = reinterpret_cast<const uint32_t*>(smem + kGMaskOff);
  uint16_t* sPos = reinterpret_cast<uint16_t*>(smem + kGPosOff);
  uint16_t* sCode = reinterpret_cast<uint16_t*>(smem + kGCodeOff);
  __shared__ __align__(8) uint64_t bar_x[2];
  __shared__ __align__(8) uint64_t bar_b;
  __shared__ __align__(8) uint64_t bar_free[2];  // every thread has gathered from buffer b
  __shared__ uint32_t tslot;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const DevTables* __restrict__ tab = a.tab;
  const int64_t grid = gridDim.x;
  const int64_t n_local = (a.n_tiles - blockIdx.x + grid - 1) / grid;  // grid <= n_tiles

  if (warp == 0) {
    tmem_alloc(&tslot, 128u);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&bar_x[0], 1);
    mbar_init(&bar_x[1], 1);
    mbar_init(&bar_b, 1);
    mbar_init(&bar_free[0], kTile);
    mbar_init(&bar_free[1], kTile);
    fence_mbar_init();
  }
  sPos[tab->chan[tid]] = static_cast<uint16_t>(tid);  // chan is a permutation of 0..127
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tlane = tslot + (static_cast<uint32_t>(warp * 32) << 16);

  if (tid == 0) {
    mbar_expect_tx(&bar_b, 256);
    bulk_g2s(smem + kGMaskOff, tab->pair_mask, 256, &bar_b);
    for (int k = 0; k < 2 && k < n_local; ++k) {
      const int row0 = static_cast<int>((blockIdx.x + k * grid) * kTile);
      mbar_expect_tx(&bar_x[k], kXBuf);
      tma_load_2d(sX + k * kXBuf, &tmap, 0, row0, &bar_x[k]);
      tma_load_2d(sX + k * kXBuf + kXBuf / 2, &tmap, 64, row0, &bar_x[k]);
    }
  }

  // store round k: this lane's natural channel 4 lane + i_k (i_k from the quantizer's
  // schedule, so that a round's 32 stores hit 32 banks) to byte offset dpos[k] of the
  // chain-ordered row, its 2 bytes taken from the lane's 8-byte load by byte permute sel[k]
  uint32_t dpos[4], sel[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint32_t i = tab->gsched[lane][k];
    dpos[k] = 2u * sPos[4 * lane + i];
    sel[k] = (2u * i) | ((2u * i + 1u) << 4);
  }
  // where those channels sit in a staged (swizzled) row: 64-column half lane / 16, 16-byte
  // chunk (lane mod 16) / 2, 8-byte half lane mod 2
  const uint32_t src_off = (lane >> 4) * (kXBuf / 2) + (lane & 1) * 8;
  const uint32_t src_c = static_cast<uint32_t>((lane & 15) >> 1);
  float thrO[NTO], thrN[NTN];
#pragma unroll
  for (int t = 0; t < NTO; ++t) thrO[t] = tab->thr[0][t];
#pragma unroll
  for (int t = 0; t < NTN; ++t) thrN[t] = tab->thr[1][t];

  bool ok = mbar_wait_ns(&bar_b, 0, kWaitNs);
  for (int64_t k = 0; k < n_local; ++k) {
    const int b = static_cast<int>(k & 1);
    const int64_t tile = blockIdx.x + k * grid;
    const int64_t row = tile * kTile + tid;
    const bool valid = row < a.n_rows;
    if (ok) ok = mbar_wait_ns(&bar_x[b], static_cast<uint32_t>((k >> 1) & 1), kWaitNs);

    // ---- gather this warp's 32 rows into chain order
    __syncwarp();  // the warp's lanes are done reading their rows of the previous tile
    {
      const uint8_t* src = sX + b * kXBuf + src_off;
#pragma unroll 4
      for (int j = 0; j < 32; ++j) {
        const int r = warp * 32 + j;
        const uint2 v = *reinterpret_cast<const uint2*>(src + r * 128 + ((src_c ^ static_cast<uint32_t>(r & 7)) << 4));
        uint8_t* dst = sP + r * kGStride;
#pragma unroll
        for (int k = 0; k < 4; ++k)
          *reinterpret_cast<uint16_t*>(dst + dpos[k]) = static_cast<uint16_t>(__byte_perm(v.x, v.y, sel[k]));
      }
    }
    mbar_arrive(&bar_free[b]);
    __syncwarp();

    // ---- own row: signs, the two norms, four 32-point transforms on (y_p, y_{p+64}) pairs
    uint64_t P[64];
    uint64_t na[4], nb[4];  // sums of squares: na pairs p < 32 (.x outliers), nb p >= 32
#pragma unroll
    for (int i = 0; i < 4; ++i) na[i] = nb[i] = pk2(0.f, 0.f);
    {
      const uint8_t* x0 = sP + tid * kGStride;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint4 u0 = *reinterpret_cast<const uint4*>(x0 + 16 * c);
        const uint4 u1 = *reinterpret_cast<const uint4*>(x0 + 128 + 16 * c);
        const uint4 m0 = *reinterpret_cast<const uint4*>(sMask + 4 * c);
        const uint4 m1 = *reinterpret_cast<const uint4*>(sMask + 32 + 4 * c);
        const uint32_t wl[4] = {u0.x ^ m0.x, u0.y ^ m0.y, u0.z ^ m0.z, u0.w ^ m0.w};
        const uint32_t wh[4] = {u1.x ^ m1.x, u1.y ^ m1.y, u1.z ^ m1.z, u1.w ^ m1.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int p = 8 * c + 2 * i;
          P[p] = pk2(__uint_as_float(wl[i] << 16), __uint_as_float(wh[i] << 16));
          P[p + 1] = pk2(__uint_as_float(wl[i] & 0xffff0000u), __uint_as_float(wh[i] & 0xffff0000u));
          if (c < 4) {
            na[i] = fma2(P[p], P[p], na[i]);
            na[i] = fma2(P[p + 1], P[p + 1], na[i]);
          } else {
            nb[i] = fma2(P[p], P[p], nb[i]);
            nb[i] = fma2(P[p + 1], P[p + 1], nb[i]);
          }
        }
      }
    }
#pragma unroll
    for (int h = 1; h < 32; h <<= 1) {
#pragma unroll
      for (int p = 0; p < 64; ++p) {
        if ((p & h) == 0) {
          const uint64_t u = P[p], v = P[p + h];
          P[p] = add2(u, v);
          P[p + h] = sub2(u, v);
        }
      }
    }
    const float2 sa = up2(add2(add2(na[0], na[1]), add2(na[2], na[3])));
    const float2 sb = up2(add2(add2(nb[0], nb[1]), add2(nb[2], nb[3])));
    const float n_o = sqrtf(sa.x), n_n = sqrtf(sa.y + (sb.x + sb.y));
    const __half no16 = __float2half_rn(n_o), nn16 = __float2half_rn(n_n);

    // ---- park the transformed row: chain position c -> TMEM column c
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      uint32_t r[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float2 v = up2(P[16 * (q & 3) + i]);
        r[i] = __float_as_uint(q < 4 ? v.x : v.y);
      }
      tmem_st16(tlane + 16 * q, r);
    }
    tmem_st_wait();

    // ---- decisions: the outlier group (2 units of 16), then the normal group (6 units)
    float TO[NTO], TN[NTN];
    const float ns = n_n * 0.57735026918962576f;  // sqrt(32 / 96)
#pragma unroll
    for (int t = 0; t < NTO; ++t) TO[t] = n_o > 0.f ? thrO[t] * n_o : thrO[t];
#pragma unroll
    for (int t = 0; t < NTN; ++t) TN[t] = n_n > 0.f ? thrN[t] * ns : thrN[t];
    // the next unit's columns are loaded while the current unit is decided
    uint32_t yA[16], yB[16];
    tmem_ld16(tlane, yA);
    tmem_ld_wait_tied16(yA);
    tmem_ld16(tlane + 16, yB);
    decide16<WO, NTO>(yA, TO, sCode, 0, tid);
    tmem_ld_wait_tied16(yB);
    tmem_ld16(tlane + 32, yA);
    decide16<WO, NTO>(yB, TO, sCode, WO, tid);
    tmem_ld_wait_tied16(yA);
#pragma unroll 1
    for (int u = 0; u < 6; u += 2) {
      tmem_ld16(tlane + 32 + 16 * (u + 1), yB);
      decide16<WN, NTN>(yA, TN, sCode, HWO + u * WN, tid);
      tmem_ld_wait_tied16(yB);
      if (u + 2 < 6) tmem_ld16(tlane + 32 + 16 * (u + 2), yA);
      decide16<WN, NTN>(yB, TN, sCode, HWO + (u + 1) * WN, tid);
      if (u + 2 < 6) tmem_ld_wait_tied16(yA);
    }

    if (valid) {
      const int64_t orow = out_row_tc(a.map, a.row_base + row);
      uint32_t w[NHW / 2];
#pragma unroll
      for (int i = 0; i < NHW / 2; ++i)
        w[i] = static_cast<uint32_t>(sCode[2 * i * kTile + tid]) |
               (static_cast<uint32_t>(sCode[(2 * i + 1) * kTile + tid]) << 16);
      uint8_t* dst = a.idx + orow * IB;
      if constexpr (IB % 16 == 0) {
#pragma unroll
        for (int i = 0; i < IB / 16; ++i)
          reinterpret_cast<uint4*>(dst)[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
      } else if constexpr (IB % 8 == 0) {
#pragma unroll
        for (int i = 0; i < IB / 8; ++i) reinterpret_cast<uint2*>(dst)[i] = make_uint2(w[2 * i], w[2 * i + 1]);
      } else {
#pragma unroll
        for (int i = 0; i < IB / 4; ++i) reinterpret_cast<uint32_t*>(dst)[i] = w[i];
      }
      a.nrm[orow * 2] = half_bits(no16);
      a.nrm[orow * 2 + 1] = half_bits(nn16);
    }

    // ---- refill staging buffer b two tiles ahead once every thread has gathered from it
    if (tid == 0 && ok && k + 2 < n_local) {
      ok = mbar_wait_ns(&bar_free[b], static_cast<uint32_t>((k >> 1) & 1), kWaitNs);
      if (ok) {
        const int row0 = static_cast<int>((tile + 2 * grid) * kTile);
        mbar_expect_tx(&bar_x[b], kXBuf);
        tma_load_2d(sX + b * kXBuf, &tmap, 0, row0, &bar_x[b]);
        tma_load_2d(sX + b * kXBuf + kXBuf / 2, &tmap, 64, row0, &bar_x[b]);
      }
    }
  }

  if (!ok) atomicOr(a.err, 1);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tslot, 128u);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

template <bool PROD, int MB>
tq_status run_tc(const CUtensorMap& tmap, const TcKeyArgs& a, cudaStream_t st) {
  auto kern = k_keys_tc<PROD, MB>;
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
  kern<<<grid, 128, kSmemBytes, st>>>(tmap, a);
  return cudaGetLastError() == cudaSuccess ? TQ_OK : TQ_ECUDA;
}

template <int B>
tq_status run_grp_tc(const CUtensorMap& tmap, const TcKeyArgs& a, cudaStream_t st) {
  auto kern = k_keys_grp_tc<B>;
  static bool attr_set = false;
  if (!attr_set) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kGSmemBytes) !=
        cudaSuccess)
      return TQ_ECUDA;
    attr_set = true;
  }
  int dev = 0;
  cudaGetDevice(&dev);
  const int64_t cap = 2ll * sm_count(dev);
  const int grid = static_cast<int>(a.n_tiles < cap ? a.n_tiles : cap);
  kern<<<grid, 128, kGSmemBytes, st>>>(tmap, a);
  return cudaGetLastError() == cudaSuccess ? TQ_OK : TQ_ECUDA;
}

}  // namespace

__device__ int g_tq_device_error = 0;

bool keys_tc_ok(const tq_quantizer* q, int dtype) {
  return dtype == TQ_BF16 && encode_fn() != nullptr;
}

tq_status launch_keys_tc(const tq_quantizer* q, const void* x, int64_t n_rows, int64_t ld,
                         tq_key_planes out, RowMap map, cudaStream_t st) {
  if (n_rows == 0) return TQ_OK;
  int* err = nullptr;
  if (cudaGetSymbolAddress(reinterpret_cast<void**>(&err), g_tq_device_error) != cudaSuccess)
    return TQ_ECUDA;
  PFN_cuTensorMapEncodeTiled_v12000 enc = encode_fn();
  if (!enc) return TQ_ECUDA;
  for (int64_t r0 = 0; r0 < n_rows; r0 += kChunkRows) {
    const int64_t nr = n_rows - r0 < kChunkRows ? n_rows - r0 : kChunkRows;
    // rows of 128 bf16 at a stride of ld elements; boxes of 64 columns x 128 rows
    CUtensorMap tmap;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(kD), static_cast<cuuint64_t>(nr)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 2};
    const cuuint32_t box[2] = {64, kTile};
    const cuuint32_t estr[2] = {1, 1};
    void* base = const_cast<uint16_t*>(static_cast<const uint16_t*>(x) + r0 * ld);
    if (enc(&tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return TQ_ECUDA;
    TcKeyArgs a{nr, r0, (nr + kTile - 1) / kTile, q->dev, out.idx, out.signs, out.norms, map, err};
    tq_status s;
    switch ((q->mode == TQ_MODE_PROD ? 8 : (q->mode == TQ_MODE_GROUPED ? 16 : 0)) + q->bits) {
      case 16 + 1: s = run_grp_tc<1>(tmap, a, st); break;
      case 16 + 2: s = run_grp_tc<2>(tmap, a, st); break;
      case 16 + 3: s = run_grp_tc<3>(tmap, a, st); break;
      case 8 + 2: s = run_tc<true, 1>(tmap, a, st); break;
      case 8 + 3: s = run_tc<true, 2>(tmap, a, st); break;
      case 8 + 4: s = run_tc<true, 3>(tmap, a, st); break;
      case 1: s = run_tc<false, 1>(tmap, a, st); break;
      case 2: s = run_tc<false, 2>(tmap, a, st); break;
      case 3: s = run_tc<false, 3>(tmap, a, st); break;
      case 4: s = run_tc<false, 4>(tmap, a, st); break;
      default: s = TQ_EUNSUPPORTED;
    }
    if (s != TQ_OK) return s;
  }
  return TQ_OK;
}

namespace {
// One thread waits on an mbarrier phase that nothing completes and gives up after limit_ns:
// the bounded-wait error path, without a device fault.
__global__ void k_selftest_wait(uint64_t limit_ns, int* err) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    if (!mbar_wait_ns(&bar, 0, limit_ns)) atomicOr(err, 1);
  }
}
}  // namespace

tq_status launch_selftest_wait(uint32_t limit_us, cudaStream_t st) {
  int* err = nullptr;
  if (cudaGetSymbolAddress(reinterpret_cast<void**>(&err), g_tq_device_error) != cudaSuccess)
    return TQ_ECUDA;
  k_selftest_wait<<<1, 32, 0, st>>>(static_cast<uint64_t>(limit_us) * 1000ull, err);
  return cudaGetLastError() == cudaSuccess ? TQ_OK : TQ_ECUDA;
}

int* device_error_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  static int* addr[64] = {};
  if (addr[dev] == nullptr) {
    int* p = nullptr;
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&p), g_tq_device_error) != cudaSuccess)
      return nullptr;
    addr[dev] = p;
  }
  return addr[dev];
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
