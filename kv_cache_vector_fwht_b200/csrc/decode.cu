// Fused decode attention over a packed prod-mode KV cache (sm_100a).
//
// Estimator (Implementing TurboQuant (part 5), algorithm overview; validate_paper.py
// attention_score):  s_i = n16_i <Pi q, c[idx_i]> + r16_i sqrt(pi/2)/d <S q, 2 sigma_i - 1>.
// With q_rot = H (s . q) (so Pi q = q_rot / sqrt(d)) and Sq = S_rot q_rot / sqrt(d):
//   <Pi q, c[idx]> = (1/d) sum_j q_rot_j C[idx_j]   (C: N(0,1)-scale centroids)
// Both sums are read from per-query lookup tables in shared memory (TurboQuant bit-packing
// article section 5: kernels consume the packed bytes directly):
//   index LUT  2-bit codes: one table per byte position p (coords 4p..4p+3), 256 entries;
//              3-bit codes in nibbles: one table per byte (coords 2p, 2p+1), 64 entries
//              addressed by lo | hi << 3; 1-bit codes: one table per nibble, 16 entries.
//   sign LUT   one table per nibble position p (coords 4p..4p+3), 16 entries of
//              sum_f Sq_{4p+f} (2 bit_f - 1).
// Entry e of table p is stored at word e * P + p (P = positions, 32 or 64), so table p lives
// in bank p mod 32. Lane l of a warp scores key l of a 32-key group and walks the positions
// starting at p = l, so the 32 lookups of one instruction hit 32 different banks.
// Tables are pre-multiplied by sm_scale * log2(e) so the online softmax runs in base 2.
//
// Grid: (context split, head group, sequence). A CTA takes one KV head, up to GC of its
// query heads, and a contiguous token range; it streams packed K/V tiles through a
// cp.async double buffer, keeps (m, l, o) per head, merges its 8 warps, and writes a partial;
// the last CTA of a (sequence, head group) to finish merges all partials (no spinning).
#include <cfloat>
#include <cmath>
#include <mutex>

#include "tq_device.cuh"
#include "tq_internal.h"

namespace tq {
namespace {

constexpr int kGC = 4;            // max query heads per CTA
constexpr int kMaxGroups = 128;
constexpr int kTile = 256;        // keys per tile (8 warps x 32)
constexpr int kThreads = 256;
constexpr int kPartStride = 132;  // floats per (head, split) partial: m, l, o[128], pad

struct DecodeArgs {
  const uint8_t* k_idx;
  const uint8_t* k_sgn;
  const uint16_t* k_nrm;
  const uint8_t* v_q;
  const uint16_t* v_par;
  const int32_t* len;
  const void* q;
  void* out;
  float* scores;
  float* part;
  int* counters;
  const DevTables* tab;
  int64_t scores_ld;
  int n_kv_heads, capacity, n_q_heads;
  int q_f32, out_f32;
  int n_splits, tokens_per_split;
  float scale_log2, inv_scale_log2;
  int16_t g_kv[kMaxGroups];
  int16_t g_heads[kMaxGroups][kGC];
  int8_t g_n[kMaxGroups];
};

template <int MB>
struct KeyGeom {
  static constexpr int IB = kD * storage_width_c(MB) / 8;           // idx bytes per key
  static constexpr int LI = MB == 1 ? 16 * 32 : (MB == 2 ? 256 * 32 : 64 * 64);  // LUT words
};

template <int MB, int VB>
struct Layout {
  static constexpr int IB = KeyGeom<MB>::IB;
  static constexpr int VQB = VB ? kD * VB / 8 : 0;
  static constexpr int VPB = VB ? 16 : 0;
  // byte offsets inside one tile stage
  static constexpr int o_idx = 0;
  static constexpr int o_sgn = o_idx + kTile * IB;
  static constexpr int o_nrm = o_sgn + kTile * 16;
  static constexpr int o_vq = o_nrm + kTile * 4;
  static constexpr int o_vp = o_vq + kTile * VQB;
  static constexpr int stage = o_vp + kTile * VPB;
  // smem regions
  static constexpr int lut_idx = 0;
  static constexpr int lut_sgn = lut_idx + kGC * KeyGeom<MB>::LI * 4;
  static constexpr int tiles = lut_sgn + kGC * 512 * 4;
  static constexpr int pbuf = tiles + 2 * stage;
  static constexpr int qbuf = pbuf + 8 * kGC * 32 * 4;    // q_rot, Sq: kGC x 2 x 128 floats
  static constexpr int total = qbuf + kGC * 2 * kD * 4;
};

template <int MB, int VB>
__device__ __forceinline__ void load_tile(uint8_t* st, const DecodeArgs& a, int64_t rowbase,
                                          int n) {
  using Lo = Layout<MB, VB>;
  // n: keys to copy (multiple of 4, within capacity)
  const int c_idx = n * Lo::IB / 16, c_sgn = n, c_nrm = n / 4;
  const int c_vq = n * Lo::VQB / 16, c_vp = VB ? n : 0;
  const int total = c_idx + c_sgn + c_nrm + c_vq + c_vp;
  for (int c = threadIdx.x; c < total; c += kThreads) {
    int r = c;
    const uint8_t* src;
    uint8_t* dst;
    if (r < c_idx) {
      src = a.k_idx + rowbase * Lo::IB + 16 * r;
      dst = st + Lo::o_idx + 16 * r;
    } else if ((r -= c_idx) < c_sgn) {
      src = a.k_sgn + rowbase * 16 + 16 * r;
      dst = st + Lo::o_sgn + 16 * r;
    } else if ((r -= c_sgn) < c_nrm) {
      src = reinterpret_cast<const uint8_t*>(a.k_nrm) + rowbase * 4 + 16 * r;
      dst = st + Lo::o_nrm + 16 * r;
    } else if ((r -= c_nrm) < c_vq) {
      src = a.v_q + rowbase * Lo::VQB + 16 * r;
      dst = st + Lo::o_vq + 16 * r;
    } else {
      r -= c_vq;
      src = reinterpret_cast<const uint8_t*>(a.v_par) + rowbase * 16 + 16 * r;
      dst = st + Lo::o_vp + 16 * r;
    }
    cp_async16(dst, src, true);
  }
}

template <int MB, int VB>
__global__ void __launch_bounds__(kThreads, 1) k_decode(const __grid_constant__ DecodeArgs a) {
  using Lo = Layout<MB, VB>;
  constexpr int IB = Lo::IB;
  constexpr int LI = KeyGeom<MB>::LI;
  constexpr bool HAS_V = VB != 0;
  extern __shared__ __align__(16) uint8_t smem[];
  float* lutI = reinterpret_cast<float*>(smem + Lo::lut_idx);
  float* lutS = reinterpret_cast<float*>(smem + Lo::lut_sgn);
  uint8_t* tiles = smem + Lo::tiles;
  float* sP = reinterpret_cast<float*>(smem + Lo::pbuf);
  float* sQ = reinterpret_cast<float*>(smem + Lo::qbuf);
  __shared__ int sLast;

  const int split = blockIdx.x, grp = blockIdx.y, b = blockIdx.z;
  const int kv = a.g_kv[grp], nh = a.g_n[grp];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int L = a.len[b];
  const int t0 = split * a.tokens_per_split;
  const int t1 = min(L, t0 + a.tokens_per_split);
  const int64_t kvrow = (static_cast<int64_t>(b) * a.n_kv_heads + kv) * a.capacity;

  float m[kGC], l[kGC], o[kGC][4];
#pragma unroll
  for (int h = 0; h < kGC; ++h) {
    m[h] = -INFINITY;
    l[h] = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) o[h][j] = 0.f;
  }

  if (t0 < t1) {
    auto tile_count = [&](int ts) {
      const int want = min(kTile, t1 - ts);
      const int n4 = (want + 3) & ~3;
      return min(n4, a.capacity - ts);
    };
    load_tile<MB, VB>(tiles, a, kvrow + t0, tile_count(t0));
    cp_async_commit();

    // ---- prologue: rotate q, project with S_rot, build the lookup tables
    const DevTables* __restrict__ tab = a.tab;
    if (warp < nh) {
      const int hq = a.g_heads[grp][warp];
      const void* qrow = a.q_f32
          ? static_cast<const void*>(static_cast<const float*>(a.q) + (static_cast<int64_t>(b) * a.n_q_heads + hq) * kD)
          : static_cast<const void*>(static_cast<const uint16_t*>(a.q) + (static_cast<int64_t>(b) * a.n_q_heads + hq) * kD);
      float v[4];
      if (a.q_f32) load4<true>(qrow, 4 * lane, v); else load4<false>(qrow, 4 * lane, v);
      const uint32_t sw = tab->sign_bits[lane >> 3];
#pragma unroll
      for (int i = 0; i < 4; ++i) v[i] = flip_sign(v[i], sw, (4 * lane + i) & 31);
      fwht_reg<4>(v);
#pragma unroll
      for (int mm = 1; mm < 32; mm <<= 1) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float other = __shfl_xor_sync(kFull, v[i], mm);
          v[i] = (lane & mm) ? (other - v[i]) : (v[i] + other);
        }
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) sQ[warp * 2 * kD + 4 * lane + i] = v[i];
    }
    __syncthreads();
    for (int e = threadIdx.x; e < nh * kD; e += kThreads) {
      const int h = e >> 7, j = e & 127;
      const float* qr = sQ + h * 2 * kD;
      float acc = 0.f;
#pragma unroll 8
      for (int i = 0; i < kD; ++i) acc = fmaf(__half2float(tab->s_rot_t[i * kD + j]), qr[i], acc);
      sQ[h * 2 * kD + kD + j] = acc * 0.088388347648318440550f;  // 1/sqrt(128)
    }
    __syncthreads();
    {
      float cen[1 << MB];
#pragma unroll
      for (int k = 0; k < (1 << MB); ++k) cen[k] = tab->cent[0][k];
      const float cI = a.scale_log2 * (1.f / 128.f);
      for (int e = threadIdx.x; e < nh * LI; e += kThreads) {
        const int h = e / LI, w = e - h * LI;
        const float* qr = sQ + h * 2 * kD;
        float val;
        if constexpr (MB == 1) {
          const int v = w >> 5, p = w & 31;
          val = 0.f;
#pragma unroll
          for (int f = 0; f < 4; ++f) val = fmaf(qr[4 * p + f], cen[(v >> f) & 1], val);
        } else if constexpr (MB == 2) {
          const int v = w >> 5, p = w & 31;
          val = 0.f;
#pragma unroll
          for (int f = 0; f < 4; ++f) val = fmaf(qr[4 * p + f], cen[(v >> (2 * f)) & 3], val);
        } else {
          const int e6 = w >> 6, p = w & 63;
          val = fmaf(qr[2 * p], cen[e6 & 7], qr[2 * p + 1] * cen[e6 >> 3]);
        }
        lutI[h * LI + w] = val * cI;
      }
      const float cS = a.scale_log2 * 1.2533141373155002512f / 128.f;  // sqrt(pi/2)/d
      for (int e = threadIdx.x; e < nh * 512; e += kThreads) {
        const int h = e >> 9, w = e & 511, v = w >> 5, p = w & 31;
        const float* sq = sQ + h * 2 * kD + kD;
        float val = 0.f;
#pragma unroll
        for (int f = 0; f < 4; ++f) val += ((v >> f) & 1) ? sq[4 * p + f] : -sq[4 * p + f];
        lutS[h * 512 + w] = val * cS;
      }
    }
    __syncthreads();

    // ---- main loop over tiles
    int it = 0;
    for (int ts = t0; ts < t1; ts += kTile, ++it) {
      uint8_t* cur = tiles + (it & 1) * Lo::stage;
      if (ts + kTile < t1)
        load_tile<MB, VB>(tiles + ((it + 1) & 1) * Lo::stage, a, kvrow + ts + kTile,
                          tile_count(ts + kTile));
      cp_async_commit();
      cp_async_wait<1>();
      __syncthreads();

      const int nk = min(kTile, t1 - ts);
      const int wcount = max(0, min(32, nk - 32 * warp));
      if (wcount > 0) {
        const int my = 32 * warp + lane;
        const bool valid = lane < wcount;
        float accI[kGC], accS[kGC];
#pragma unroll
        for (int h = 0; h < kGC; ++h) { accI[h] = 0.f; accS[h] = 0.f; }

        // index term
        if constexpr (MB == 2) {
          const uint32_t* kr = reinterpret_cast<const uint32_t*>(cur + Lo::o_idx + my * IB);
          const int q = lane >> 2, sh = 8 * (lane & 3);
          uint32_t w[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) w[i] = kr[(q + i) & 7];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const uint32_t R = __funnelshift_r(w[i], w[(i + 1) & 7], sh);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const uint32_t v = (R >> (8 * k)) & 0xffu;
              const float* Lp = lutI + (v << 5) + ((lane + 4 * i + k) & 31);
#pragma unroll
              for (int h = 0; h < kGC; ++h)
                if (h < nh) accI[h] += Lp[h * LI];
            }
          }
        } else if constexpr (MB == 3) {
          const uint32_t* kr = reinterpret_cast<const uint32_t*>(cur + Lo::o_idx + my * IB);
          const int q = lane >> 2, sh = 8 * (lane & 3);
          uint32_t w[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) w[i] = kr[(q + i) & 15];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const uint32_t R = __funnelshift_r(w[i], w[(i + 1) & 15], sh);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const uint32_t v = (R >> (8 * k)) & 0xffu;
              const uint32_t e6 = (v & 7u) | ((v >> 1) & 0x38u);
              const float* Lp = lutI + (e6 << 6) + ((lane + 4 * i + k) & 63);
#pragma unroll
              for (int h = 0; h < kGC; ++h)
                if (h < nh) accI[h] += Lp[h * LI];
            }
          }
        } else {  // MB == 1: nibble tables over 16 index bytes
          const uint32_t* kr = reinterpret_cast<const uint32_t*>(cur + Lo::o_idx + my * IB);
          const int q = lane >> 3, sh = 4 * (lane & 7);
          uint32_t w[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) w[i] = kr[(q + i) & 3];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint32_t R = __funnelshift_r(w[i], w[(i + 1) & 3], sh);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const uint32_t v = (R >> (4 * k)) & 0xfu;
              const float* Lp = lutI + (v << 5) + ((lane + 8 * i + k) & 31);
#pragma unroll
              for (int h = 0; h < kGC; ++h)
                if (h < nh) accI[h] += Lp[h * LI];
            }
          }
        }
        // QJL sign term (nibble tables over the 16 sign bytes)
        {
          const uint32_t* sr = reinterpret_cast<const uint32_t*>(cur + Lo::o_sgn + my * 16);
          const int q = lane >> 3, sh = 4 * (lane & 7);
          uint32_t w[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) w[i] = sr[(q + i) & 3];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint32_t R = __funnelshift_r(w[i], w[(i + 1) & 3], sh);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const uint32_t v = (R >> (4 * k)) & 0xfu;
              const float* Lp = lutS + (v << 5) + ((lane + 8 * i + k) & 31);
#pragma unroll
              for (int h = 0; h < kGC; ++h)
                if (h < nh) accS[h] += Lp[h * 512];
            }
          }
        }
        const uint32_t nn = reinterpret_cast<const uint32_t*>(cur + Lo::o_nrm)[my];
        const float n16 = half_lo(nn), r16 = half_hi(nn);

        float p[kGC];
#pragma unroll
        for (int h = 0; h < kGC; ++h) {
          if (h < nh) {
            const float s = valid ? fmaf(n16, accI[h], r16 * accS[h]) : -INFINITY;
            if (a.scores != nullptr && valid) {
              const int hq = a.g_heads[grp][h];
              a.scores[(static_cast<int64_t>(b) * a.n_q_heads + hq) * a.scores_ld + ts + my] =
                  s * a.inv_scale_log2;
            }
            if constexpr (HAS_V) {
              const float mx = warp_max(s);
              const float mn = fmaxf(m[h], mx);
              const float alpha = exp2f(m[h] - mn);
              p[h] = exp2f(s - mn);
              l[h] = fmaf(l[h], alpha, p[h]);
#pragma unroll
              for (int j = 0; j < 4; ++j) o[h][j] *= alpha;
              m[h] = mn;
              sP[(warp * kGC + h) * 32 + lane] = p[h];
            }
          }
        }
        if constexpr (HAS_V) {
          __syncwarp();
          const int g = lane >> 3;
          for (int i = 0; i < wcount; ++i) {
            const int key = 32 * warp + i;
            const uint32_t par = reinterpret_cast<const uint32_t*>(cur + Lo::o_vp + key * 16)[g];
            const float mnv = half_lo(par), scv = half_hi(par);
            float vv[4];
            if constexpr (VB == 2) {
              const uint32_t by = cur[Lo::o_vq + key * 32 + lane];
#pragma unroll
              for (int j = 0; j < 4; ++j) vv[j] = fmaf(static_cast<float>((by >> (2 * j)) & 3u), scv, mnv);
            } else {
              const uint32_t hw = reinterpret_cast<const uint16_t*>(cur + Lo::o_vq + key * 64)[lane];
#pragma unroll
              for (int j = 0; j < 4; ++j) vv[j] = fmaf(static_cast<float>((hw >> (4 * j)) & 15u), scv, mnv);
            }
#pragma unroll
            for (int h = 0; h < kGC; ++h) {
              if (h < nh) {
                const float ph = sP[(warp * kGC + h) * 32 + i];
#pragma unroll
                for (int j = 0; j < 4; ++j) o[h][j] = fmaf(ph, vv[j], o[h][j]);
              }
            }
          }
          __syncwarp();
        }
      }
      __syncthreads();
    }
    cp_async_wait<0>();
  }

  if constexpr (!HAS_V) return;

  // ---- merge the 8 warps of this CTA (reusing the tile buffers)
  __syncthreads();
  float* sM = reinterpret_cast<float*>(tiles);  // [warp][h][kPartStride]
#pragma unroll
  for (int h = 0; h < kGC; ++h) {
    if (h < nh) {
      const float lt = warp_sum(l[h]);
      float* dst = sM + (warp * kGC + h) * kPartStride;
      if (lane == 0) { dst[0] = m[h]; dst[1] = lt; }
#pragma unroll
      for (int j = 0; j < 4; ++j) dst[2 + 4 * lane + j] = o[h][j];
    }
  }
  __syncthreads();
  if (warp < nh) {
    const int h = warp, hq = a.g_heads[grp][h];
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < 8; ++w) M = fmaxf(M, sM[(w * kGC + h) * kPartStride]);
    float Lsum = 0.f, O[4] = {0.f, 0.f, 0.f, 0.f};
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < 8; ++w) {
        const float* src = sM + (w * kGC + h) * kPartStride;
        const float f = exp2f(src[0] - M);
        Lsum = fmaf(f, src[1], Lsum);
#pragma unroll
        for (int j = 0; j < 4; ++j) O[j] = fmaf(f, src[2 + 4 * lane + j], O[j]);
      }
    }
    const int64_t orow = (static_cast<int64_t>(b) * a.n_q_heads + hq) * kD + 4 * lane;
    if (a.n_splits == 1) {
      const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
      if (a.out_f32) {
        *reinterpret_cast<float4*>(static_cast<float*>(a.out) + orow) =
            make_float4(O[0] * inv, O[1] * inv, O[2] * inv, O[3] * inv);
      } else {
        __nv_bfloat162 lo = __floats2bfloat162_rn(O[0] * inv, O[1] * inv);
        __nv_bfloat162 hi = __floats2bfloat162_rn(O[2] * inv, O[3] * inv);
        uint2 pk;
        pk.x = *reinterpret_cast<uint32_t*>(&lo);
        pk.y = *reinterpret_cast<uint32_t*>(&hi);
        *reinterpret_cast<uint2*>(static_cast<uint16_t*>(a.out) + orow) = pk;
      }
    } else {
      float* dst = a.part + ((static_cast<int64_t>(b) * a.n_q_heads + hq) * a.n_splits + split) * kPartStride;
      if (lane == 0) { dst[0] = M; dst[1] = Lsum; }
      *reinterpret_cast<float4*>(dst + 4 + 4 * lane) = make_float4(O[0], O[1], O[2], O[3]);
    }
  }
  if (a.n_splits == 1) return;

  // ---- the last CTA of this (sequence, head group) merges all splits
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    int* ctr = a.counters + static_cast<int64_t>(b) * a.n_q_heads + a.g_heads[grp][0];
    sLast = atomicAdd(ctr, 1) == a.n_splits - 1;
  }
  __syncthreads();
  if (!sLast) return;
  __threadfence();
  if (warp < nh) {
    const int h = warp, hq = a.g_heads[grp][h];
    const float* base = a.part + (static_cast<int64_t>(b) * a.n_q_heads + hq) * a.n_splits * kPartStride;
    float M = -INFINITY;
    for (int s = 0; s < a.n_splits; ++s) M = fmaxf(M, __ldcg(base + s * kPartStride));
    float Lsum = 0.f, O[4] = {0.f, 0.f, 0.f, 0.f};
    if (M != -INFINITY) {
      for (int s = 0; s < a.n_splits; ++s) {
        const float* src = base + s * kPartStride;
        const float ms = __ldcg(src);
        if (ms == -INFINITY) continue;
        const float f = exp2f(ms - M);
        Lsum = fmaf(f, __ldcg(src + 1), Lsum);
        const float4 ov = __ldcg(reinterpret_cast<const float4*>(src + 4 + 4 * lane));
        O[0] = fmaf(f, ov.x, O[0]);
        O[1] = fmaf(f, ov.y, O[1]);
        O[2] = fmaf(f, ov.z, O[2]);
        O[3] = fmaf(f, ov.w, O[3]);
      }
    }
    const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
    const int64_t orow = (static_cast<int64_t>(b) * a.n_q_heads + hq) * kD + 4 * lane;
    if (a.out_f32) {
      *reinterpret_cast<float4*>(static_cast<float*>(a.out) + orow) =
          make_float4(O[0] * inv, O[1] * inv, O[2] * inv, O[3] * inv);
    } else {
      __nv_bfloat162 lo = __floats2bfloat162_rn(O[0] * inv, O[1] * inv);
      __nv_bfloat162 hi = __floats2bfloat162_rn(O[2] * inv, O[3] * inv);
      uint2 pk;
      pk.x = *reinterpret_cast<uint32_t*>(&lo);
      pk.y = *reinterpret_cast<uint32_t*>(&hi);
      *reinterpret_cast<uint2*>(static_cast<uint16_t*>(a.out) + orow) = pk;
    }
  }
  if (threadIdx.x == 0) a.counters[static_cast<int64_t>(b) * a.n_q_heads + a.g_heads[grp][0]] = 0;
}

template <int MB, int VB>
tq_status run_decode(const DecodeArgs& a, dim3 grid, cudaStream_t st) {
  constexpr int smem = Layout<MB, VB>::total;
  static_assert(smem <= 227 * 1024, "decode shared memory budget");
  auto kern = k_decode<MB, VB>;
  static bool configured = false;
  if (!configured) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
        cudaSuccess)
      return TQ_ECUDA;
    configured = true;
  }
  kern<<<grid, kThreads, smem, st>>>(a);
  return cudaGetLastError() == cudaSuccess ? TQ_OK : TQ_ECUDA;
}

int max_splits_for(int capacity) {
  const int s = (capacity + kTile - 1) / kTile;
  return s < 1 ? 1 : (s > 256 ? 256 : s);
}

}  // namespace

size_t decode_workspace_bytes(int batch, int n_q_heads, int capacity) {
  const size_t parts = static_cast<size_t>(batch) * n_q_heads * max_splits_for(capacity) *
                       kPartStride * sizeof(float);
  const size_t ctrs = static_cast<size_t>(batch) * n_q_heads * sizeof(int);
  return ((parts + 255) / 256) * 256 + ((ctrs + 255) / 256) * 256;
}

tq_status launch_decode(const tq_quantizer* q, const tq_kv_cache* c, const void* qv, int q_dtype,
                        int n_q_heads, const int32_t* head_map, float sm_scale, void* out,
                        int out_dtype, float* scores, int64_t scores_ld, void* workspace,
                        size_t workspace_bytes, cudaStream_t st) {
  DecodeArgs a{};
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
  a.n_kv_heads = c->n_kv_heads;
  a.capacity = c->capacity;
  a.n_q_heads = n_q_heads;
  a.q_f32 = q_dtype == TQ_F32;
  a.out_f32 = out_dtype == TQ_F32;
  const float scale = sm_scale > 0.f ? sm_scale : 1.f / std::sqrt(static_cast<float>(kD));
  a.scale_log2 = scale * 1.4426950408889634074f;
  a.inv_scale_log2 = 1.f / a.scale_log2;

  // head groups: the query heads of each KV head, in up to kGC-sized balanced groups
  int n_groups = 0;
  for (int kv = 0; kv < c->n_kv_heads; ++kv) {
    int heads[1024];
    int n = 0;
    for (int h = 0; h < n_q_heads; ++h)
      if ((head_map ? head_map[h] : h / (n_q_heads / c->n_kv_heads)) == kv) heads[n++] = h;
    if (n == 0) continue;
    const int ng = (n + kGC - 1) / kGC;
    int pos = 0;
    for (int g = 0; g < ng; ++g) {
      const int cnt = (n - pos) / (ng - g);
      if (n_groups >= kMaxGroups) return TQ_EUNSUPPORTED;
      a.g_kv[n_groups] = static_cast<int16_t>(kv);
      a.g_n[n_groups] = static_cast<int8_t>(cnt);
      for (int i = 0; i < cnt; ++i) a.g_heads[n_groups][i] = static_cast<int16_t>(heads[pos + i]);
      pos += cnt;
      ++n_groups;
    }
  }
  if (n_groups == 0) return TQ_OK;

  int max_len = 0;
  for (int b = 0; b < c->batch; ++b) max_len = c->len_host[b] > max_len ? c->len_host[b] : max_len;
  if (max_len == 0 && out == nullptr) return TQ_OK;

  // split count: minimise waves x (tokens per split + per-CTA set-up), one CTA per SM
  int dev = 0;
  cudaGetDevice(&dev);
  const int sms = sm_count(dev);
  const int pairs = c->batch * n_groups;
  const int cap_splits = max_splits_for(c->capacity);
  int best = 1;
  double best_cost = 1e300;
  const int max_try = std::max(1, std::min(cap_splits, (max_len + kTile - 1) / kTile));
  for (int s = 1; s <= max_try; ++s) {
    const int tps = ((max_len + s - 1) / s + 31) & ~31;
    const int used = (max_len + tps - 1) / tps;
    if (used != s) continue;
    const double waves = std::ceil(static_cast<double>(pairs) * s / sms);
    const double cost = waves * (tps + 512.0);
    if (cost < best_cost - 1e-9) { best_cost = cost; best = s; }
  }
  a.n_splits = best;
  a.tokens_per_split = std::max(32, ((max_len + best - 1) / best + 31) & ~31);
  if (decode_workspace_bytes(c->batch, n_q_heads, c->capacity) > workspace_bytes) return TQ_EINVAL;
  const size_t parts = static_cast<size_t>(c->batch) * n_q_heads * cap_splits * kPartStride * sizeof(float);
  a.part = static_cast<float*>(workspace);
  a.counters = reinterpret_cast<int*>(static_cast<uint8_t*>(workspace) + ((parts + 255) / 256) * 256);

  const dim3 grid(a.n_splits, n_groups, c->batch);
  const int mb = q->bits - 1;
  const int vb = c->value_bits;
  switch (mb * 8 + vb) {
    case 1 * 8 + 0: return run_decode<1, 0>(a, grid, st);
    case 1 * 8 + 2: return run_decode<1, 2>(a, grid, st);
    case 1 * 8 + 4: return run_decode<1, 4>(a, grid, st);
    case 2 * 8 + 0: return run_decode<2, 0>(a, grid, st);
    case 2 * 8 + 2: return run_decode<2, 2>(a, grid, st);
    case 2 * 8 + 4: return run_decode<2, 4>(a, grid, st);
    case 3 * 8 + 0: return run_decode<3, 0>(a, grid, st);
    case 3 * 8 + 2: return run_decode<3, 2>(a, grid, st);
    case 3 * 8 + 4: return run_decode<3, 4>(a, grid, st);
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
                       scores_ld, base, need, st);
}

}  // namespace tq
