// Fused decode attention over a packed prod-mode KV cache (sm_100a).
//
// Estimator (Implementing TurboQuant (part 5), algorithm overview; validate_paper.py
// attention_score):  s_i = n16_i <Pi q, c[idx_i]> + r16_i sqrt(pi/2)/d <S q, 2 sigma_i - 1>.
// With q_rot = H (s . q) (so Pi q = q_rot / sqrt(d)) and Sq = S_rot q_rot / sqrt(d):
//   <Pi q, c[idx]> = (1/d) sum_j q_rot_j C[idx_j]      (C: N(0,1)-scale centroids).
// Both sums are read from per-query lookup tables in shared memory; the kernel consumes the
// packed bytes directly (TurboQuant bit-packing article, section 5).
//
// Lookup tables. A field is the packed bits covering consecutive coordinates: a 2-bit index
// byte (4 coordinates), a byte of two 3-bit indices in nibbles (2 coordinates), a 1-bit index
// nibble (4 coordinates) or a QJL sign nibble (4 coordinates). The Lloyd-Max codebook is
// symmetric (C[L-1-k] = -C[k]) and the sign sums are odd, so the value of a field and of its
// mirror (all codes k -> L-1-k, all signs flipped) differ only in sign: a table keeps the
// canonical half of the fields (top code bit clear) and a lookup returns (entry, +-1).
// Entries hold 4 query heads (16 bytes); 8 heads use two such tables. Entry e of position p
// sits at ((e * P + p) * 16) bytes, so position p lives in bank group p mod 8 and the eight
// lanes of one 16-byte shared-memory phase (walking positions p = lane + s) never collide.
// Tables are pre-multiplied by sm_scale * log2(e): the online softmax runs in base 2.
//
// Grid: (context split, head group, sequence). A CTA takes one KV head, up to 8 of its query
// heads and a contiguous token range; it streams packed K/V tiles of 256 tokens through a
// cp.async double buffer; lane l of warp w scores token 32w + l; then lanes split the 128
// channels of P.V (8 per lane, two tokens per step) with packed fp32x2 FMAs. Each CTA merges
// its warps and writes a partial (m, l, o); the last CTA of a (sequence, head group) to
// finish merges all partials (an atomic counter, no waiting).
#include <cfloat>
#include <cmath>
#include <mutex>

#include "tq_device.cuh"
#include "tq_internal.h"

namespace tq {
namespace {

constexpr int kMaxHeads = 8;      // query heads per CTA
constexpr int kMaxGroups = 128;
constexpr int kTile = 256;        // tokens per tile (8 warps x 32)
constexpr int kThreads = 256;
constexpr int kPartStride = 132;  // floats per (head, split) partial: m, l, pad, o[128]
constexpr int kSrotStride = 272;  // bytes per staged S_rot row (256 + 16: bank spread)

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
  int16_t g_heads[kMaxGroups][kMaxHeads];
  int8_t g_n[kMaxGroups];
};

// (+1.0, +1.0) or (-1.0, -1.0) from an all-ones / all-zeros mask
__device__ __forceinline__ uint64_t sign_pair(int mask) {
  const float s = __uint_as_float(0x3f800000u | (static_cast<uint32_t>(mask) & 0x80000000u));
  return pk2(s, s);
}

// Shared-memory plan. A table has P positions of E canonical 16-byte entries (4 heads);
// positions are stored P + 32 times wide where noted (entry p + P repeats entry p) so that
// lane l's walk p = l + s never wraps and s becomes an immediate load offset.
template <int MB, int VB, int NH4>
struct Lay {
  static constexpr int IB = kD * storage_width_c(MB) / 8;            // index bytes per token
  static constexpr bool NIB = MB != 3;                               // nibble index tables
  static constexpr int PI = MB == 2 ? 64 : (MB == 1 ? 32 : 64);      // index positions
  static constexpr int EI = MB == 3 ? 32 : 8;                        // canonical entries
  static constexpr int PDI = NIB ? PI + 32 : PI;                     // stored positions
  static constexpr int HALF_I = EI * PDI * 16;
  static constexpr int PDS = 64;                                     // sign table, stored
  static constexpr int HALF_S = 8 * PDS * 16;
  static constexpr int STAGES = MB == 3 ? 2 : 1;
  static constexpr int VQB = VB ? kD * VB / 8 : 0;
  static constexpr int VPB = VB ? 16 : 0;
  // one tile stage
  static constexpr int o_idx = 0;
  static constexpr int o_sgn = o_idx + kTile * IB;
  static constexpr int o_nrm = o_sgn + kTile * 16;
  static constexpr int o_vq = o_nrm + kTile * 4;
  static constexpr int o_vp = o_vq + kTile * VQB;
  static constexpr int stage = o_vp + kTile * VPB;
  // regions: tables, query buffers,
  // tile stages, then per-warp p pairs and dequant pairs (tiles..end reused for the merge)
  static constexpr int lut_bytes = NH4 * (HALF_I + HALF_S);
  static constexpr int lutI = 0;
  static constexpr int lutS = NH4 * HALF_I;
  static constexpr int qrT = (lut_bytes + 127) & ~127;               // q_rot [128][8] f32
  static constexpr int sqT = qrT + kD * kMaxHeads * 4;               // Sq    [128][8] f32
  static constexpr int qhi = sqT + kD * kMaxHeads * 4;               // hi [8][136] f16
  static constexpr int qlo = qhi + kMaxHeads * kSrotStride;          // lo [8][136] f16
  static constexpr int qinv = qlo + kMaxHeads * kSrotStride;         // [8] f32
  static constexpr int tiles = (qinv + 32 + 127) & ~127;
  static constexpr int ppair = tiles + STAGES * stage;               // [8][32][8] (p, p)
  static constexpr int vpair = ppair + 8 * 32 * kMaxHeads * 8;       // [8][32][4] (s16,s16,c,c)
  static constexpr int end_v = vpair + (VB ? 8 * 32 * 4 * 16 : 0);
  static constexpr int merge = 8 * kMaxHeads * kPartStride * 4;
  static constexpr int total = (end_v - tiles) >= merge ? end_v : tiles + merge;
};

template <int MB, int VB, int NH4>
__device__ __forceinline__ void load_tile(uint8_t* st, const DecodeArgs& a, int64_t rowbase,
                                          int n) {
  using Lo = Lay<MB, VB, NH4>;
  // n: tokens to copy (a multiple of 4, within capacity)
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

// Accumulate one 4-head (or 8-head) table entry with sign: acc[j] += sg * entry.
template <int NH4, int HALF>
__device__ __forceinline__ void lut_acc(uint64_t (&acc)[4], const uint8_t* p, uint64_t sg) {
  const ulonglong2 L = *reinterpret_cast<const ulonglong2*>(p);
  acc[0] = fma2(sg, L.x, acc[0]);
  acc[1] = fma2(sg, L.y, acc[1]);
  if constexpr (NH4 == 2) {
    const ulonglong2 M = *reinterpret_cast<const ulonglong2*>(p + HALF);
    acc[2] = fma2(sg, M.x, acc[2]);
    acc[3] = fma2(sg, M.y, acc[3]);
  }
}

// Nibble-table lookup for nibble s of the lane-rotated words R (field sign-extended from its
// top bit: negative fields use the mirrored canonical entry with sign -1).
template <int NH4, int HALF, int STRIDE>
__device__ __forceinline__ void nib_step(uint64_t (&acc)[4], uint32_t w, int k, const uint8_t* lane_base,
                                         int s) {
  const int t = static_cast<int>(w << (28 - 4 * k)) >> 28;
  const int msk = t >> 31;
  const uint8_t* p = lane_base + (t ^ msk) * STRIDE + 16 * s;
  lut_acc<NH4, HALF>(acc, p, sign_pair(msk));
}

template <int MB, int VB, int NH4>
__global__ void __launch_bounds__(kThreads, MB == 3 ? 1 : 2)
k_decode(const __grid_constant__ DecodeArgs a) {
  using Lo = Lay<MB, VB, NH4>;
  constexpr int IB = Lo::IB, PI = Lo::PI, EI = Lo::EI, PDI = Lo::PDI;
  constexpr int NH = 4 * NH4;
  constexpr bool HAS_V = VB != 0;
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* lutI = smem + Lo::lutI;
  uint8_t* lutS = smem + Lo::lutS;
  float* qrT = reinterpret_cast<float*>(smem + Lo::qrT);
  float* sqT = reinterpret_cast<float*>(smem + Lo::sqT);
  uint8_t* qhi = smem + Lo::qhi;
  uint8_t* qlo = smem + Lo::qlo;
  float* qinv = reinterpret_cast<float*>(smem + Lo::qinv);
  uint8_t* tiles = smem + Lo::tiles;
  __shared__ int sLast;
  __shared__ float sCen[16];

  const int split = blockIdx.x, grp = blockIdx.y, b = blockIdx.z;
  const int kv = a.g_kv[grp], nh = a.g_n[grp];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int L = a.len[b];
  const int t0 = split * a.tokens_per_split;
  const int t1 = min(L, t0 + a.tokens_per_split);
  const int64_t kvrow = (static_cast<int64_t>(b) * a.n_kv_heads + kv) * a.capacity;

  float m[NH], l[NH];
  uint64_t o[NH][2];   // channels (4 lane, 4 lane + 1), (4 lane + 2, 4 lane + 3)
#pragma unroll
  for (int h = 0; h < NH; ++h) {
    m[h] = -INFINITY;
    l[h] = 0.f;
    o[h][0] = 0ull;
    o[h][1] = 0ull;
  }

  if (t0 < t1) {
    auto tile_count = [&](int ts) {
      const int want = min(kTile, t1 - ts);
      const int n4 = (want + 3) & ~3;
      return min(n4, a.capacity - ts);
    };
    load_tile<MB, VB, NH4>(tiles, a, kvrow + t0, tile_count(t0));
    cp_async_commit();

    // ---------------- prologue (b1): rotate q, project with S_rot, build the tables
    const DevTables* __restrict__ tab = a.tab;
    // this warp's S_rot rows [16 warp, 16 warp + 16) as mma.sync A fragments, read from L2
    uint32_t afr[8][4];
    {
      const int g = lane >> 2, t = lane & 3;
      const uint32_t* r0 = reinterpret_cast<const uint32_t*>(tab->s_rot + (16 * warp + g) * kD);
      const uint32_t* r1 = r0 + 8 * kD / 2;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        afr[kk][0] = __ldg(r0 + kk * 8 + t);
        afr[kk][1] = __ldg(r1 + kk * 8 + t);
        afr[kk][2] = __ldg(r0 + kk * 8 + 4 + t);
        afr[kk][3] = __ldg(r1 + kk * 8 + 4 + t);
      }
    }
    {
      // q_rot of head `warp` (zeros for padded heads): signs, then the 128-point transform
      // with 4 values per lane (2 stages in registers, 5 across lanes)
      float v[4] = {0.f, 0.f, 0.f, 0.f};
      if (warp < nh) {
        const int hq = a.g_heads[grp][warp];
        const int64_t qoff = (static_cast<int64_t>(b) * a.n_q_heads + hq) * kD;
        if (a.q_f32) load4<true>(static_cast<const float*>(a.q) + qoff, 4 * lane, v);
        else load4<false>(static_cast<const uint16_t*>(a.q) + qoff, 4 * lane, v);
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
      }
      // power-of-two scale so the fp16 hi/lo split neither overflows nor underflows
      float amax = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
      amax = warp_max(amax);
      const uint32_t ex = (__float_as_uint(amax) >> 23) & 0xffu;
      const bool big = ex >= 12u;
      const float scl = big ? __uint_as_float((264u - ex) << 23) : 1.f;
      const float inv = big ? __uint_as_float((ex - 10u) << 23) : 1.f;
      if (lane == 0) qinv[warp] = inv;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int j = 4 * lane + i;
        qrT[j * kMaxHeads + warp] = v[i];
        const float sv = v[i] * scl;
        const __half hi = __float2half_rn(sv);
        const __half lo = __float2half_rn(sv - __half2float(hi));
        reinterpret_cast<__half*>(qhi + warp * kSrotStride)[j] = hi;
        reinterpret_cast<__half*>(qlo + warp * kSrotStride)[j] = lo;
      }
    }
    if (threadIdx.x < 16) sCen[threadIdx.x] = tab->cent[0][threadIdx.x];
    __syncthreads();
    {
      // Sq = S_rot q_rot / sqrt(d) for the 8 head slots on tensor cores: mma.sync m16n8k16
      // (fp16 S_rot is exact; q_rot enters as hi + lo fp16 halves; fp32 accumulation).
      const int g = lane >> 2, t = lane & 3;
      float c0 = 0.f, c1 = 0.f, c2 = 0.f, c3 = 0.f;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const int k0 = 16 * kk;
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          const uint8_t* bq = (part ? qlo : qhi) + g * kSrotStride;
          const uint32_t b0 = *reinterpret_cast<const uint32_t*>(bq + (k0 + 2 * t) * 2);
          const uint32_t b1 = *reinterpret_cast<const uint32_t*>(bq + (k0 + 8 + 2 * t) * 2);
          asm volatile(
              "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
              "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};\n"
              : "+f"(c0), "+f"(c1), "+f"(c2), "+f"(c3)
              : "r"(afr[kk][0]), "r"(afr[kk][1]), "r"(afr[kk][2]), "r"(afr[kk][3]), "r"(b0), "r"(b1));
        }
      }
      const float s0 = qinv[2 * t] * 0.088388347648318440550f;      // / sqrt(128)
      const float s1 = qinv[2 * t + 1] * 0.088388347648318440550f;
      const int j0 = 16 * warp + g;
      sqT[j0 * kMaxHeads + 2 * t] = c0 * s0;
      sqT[j0 * kMaxHeads + 2 * t + 1] = c1 * s1;
      sqT[(j0 + 8) * kMaxHeads + 2 * t] = c2 * s0;
      sqT[(j0 + 8) * kMaxHeads + 2 * t + 1] = c3 * s1;
    }
    __syncthreads();
    {
      const float* cen = sCen;
      const float cI = a.scale_log2 * (1.f / 128.f);
      const float cS = a.scale_log2 * 1.2533141373155002512f / 128.f;  // sqrt(pi/2) / d
      // index tables: one thread per (4-head half, stored position), all entries of it
      for (int e = threadIdx.x; e < NH4 * PDI; e += kThreads) {
        const int hf = e / PDI, pd = e - hf * PDI;
        const int p = pd < PI ? pd : pd - PI;
        uint8_t* dst = lutI + hf * Lo::HALF_I + pd * 16;
        if constexpr (MB == 1) {          // nibble: four 1-bit codes (C = -c, +c), coords 4p..4p+3
          const float c = cen[1] * cI;
          float4 x[4];
#pragma unroll
          for (int f = 0; f < 4; ++f) x[f] = *reinterpret_cast<const float4*>(qrT + (4 * p + f) * kMaxHeads + 4 * hf);
#pragma unroll
          for (int en = 0; en < 8; ++en) {
            float4 r = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int f = 0; f < 4; ++f) {
              const float sg = ((en >> f) & 1) ? c : -c;
              r.x = fmaf(x[f].x, sg, r.x); r.y = fmaf(x[f].y, sg, r.y);
              r.z = fmaf(x[f].z, sg, r.z); r.w = fmaf(x[f].w, sg, r.w);
            }
            *reinterpret_cast<float4*>(dst + en * PDI * 16) = r;
          }
        } else {                          // two codes (2-bit nibble or 3-bit byte), coords 2p, 2p+1
          const float4 x = *reinterpret_cast<const float4*>(qrT + (2 * p) * kMaxHeads + 4 * hf);
          const float4 y = *reinterpret_cast<const float4*>(qrT + (2 * p + 1) * kMaxHeads + 4 * hf);
          constexpr int LO = MB == 2 ? 4 : 8;     // levels of the first code
#pragma unroll
          for (int en = 0; en < EI; ++en) {
            const float c0 = cen[en % LO] * cI, c1 = cen[en / LO] * cI;
            *reinterpret_cast<float4*>(dst + en * PDI * 16) =
                make_float4(fmaf(x.x, c0, y.x * c1), fmaf(x.y, c0, y.y * c1),
                            fmaf(x.z, c0, y.z * c1), fmaf(x.w, c0, y.w * c1));
          }
        }
      }
      // QJL sign tables: entry bit f = sign bit of coordinate 4p + f (+1 if set, else -1)
      for (int e = threadIdx.x; e < NH4 * Lo::PDS; e += kThreads) {
        const int hf = e / Lo::PDS, pd = e - hf * Lo::PDS, p = pd & 31;
        float4 x[4];
#pragma unroll
        for (int f = 0; f < 4; ++f) x[f] = *reinterpret_cast<const float4*>(sqT + (4 * p + f) * kMaxHeads + 4 * hf);
        uint8_t* dst = lutS + hf * Lo::HALF_S + pd * 16;
#pragma unroll
        for (int en = 0; en < 8; ++en) {
          float4 r = make_float4(-x[3].x * cS, -x[3].y * cS, -x[3].z * cS, -x[3].w * cS);
#pragma unroll
          for (int f = 0; f < 3; ++f) {
            const float sg = ((en >> f) & 1) ? cS : -cS;
            r.x = fmaf(x[f].x, sg, r.x); r.y = fmaf(x[f].y, sg, r.y);
            r.z = fmaf(x[f].z, sg, r.z); r.w = fmaf(x[f].w, sg, r.w);
          }
          *reinterpret_cast<float4*>(dst + en * Lo::PDS * 16) = r;
        }
      }
    }
    __syncthreads();

    // ---------------- main loop over tiles (b2-b4)
    uint64_t* sPP = reinterpret_cast<uint64_t*>(smem + Lo::ppair) + warp * 32 * kMaxHeads;
    float4* sVP = reinterpret_cast<float4*>(smem + Lo::vpair) + warp * 32 * 4;
    int it = 0;
    for (int ts = t0; ts < t1; ts += kTile, ++it) {
      uint8_t* cur = tiles + (Lo::STAGES == 2 ? (it & 1) * Lo::stage : 0);
      if constexpr (Lo::STAGES == 2) {
        if (ts + kTile < t1)
          load_tile<MB, VB, NH4>(tiles + ((it + 1) & 1) * Lo::stage, a, kvrow + ts + kTile,
                                 tile_count(ts + kTile));
        cp_async_commit();
        cp_async_wait<1>();
      } else {
        if (it > 0) {
          load_tile<MB, VB, NH4>(tiles, a, kvrow + ts, tile_count(ts));
          cp_async_commit();
        }
        cp_async_wait<0>();
      }
      __syncthreads();

      const int nk = min(kTile, t1 - ts);
      const int wcount = max(0, min(32, nk - 32 * warp));
      if (wcount > 0) {
        const int my = 32 * warp + lane;
        const bool valid = lane < wcount;
        uint64_t accI[4] = {0ull, 0ull, 0ull, 0ull}, accS[4] = {0ull, 0ull, 0ull, 0ull};
        // sign nibbles, rotated by `lane` nibbles: nibble k of RS[i] = (lane + 8i + k) mod 32
        {
          const uint32_t* sr = reinterpret_cast<const uint32_t*>(cur + Lo::o_sgn + my * 16);
          const int q = lane >> 3, sh = 4 * (lane & 7);
          uint32_t w[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) w[i] = sr[(q + i) & 3];
          const uint8_t* lb = lutS + lane * 16;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint32_t R = __funnelshift_r(w[i], w[(i + 1) & 3], sh);
#pragma unroll
            for (int k = 0; k < 8; ++k)
              nib_step<NH4, Lo::HALF_S, Lo::PDS * 16>(accS, R, k, lb, 8 * i + k);
          }
        }
        if constexpr (MB == 2 || MB == 1) {
          // index nibbles, rotated by `lane` nibbles
          constexpr int NW = IB / 4;       // 8 words (2-bit) or 4 words (1-bit)
          const uint32_t* kr = reinterpret_cast<const uint32_t*>(cur + Lo::o_idx + my * IB);
          const int q = lane >> 3, sh = 4 * (lane & 7);
          uint32_t w[NW];
#pragma unroll
          for (int i = 0; i < NW; ++i) w[i] = kr[(q + i) % NW];
          const uint8_t* lb = lutI + lane * 16;
#pragma unroll
          for (int i = 0; i < NW; ++i) {
            const uint32_t R = __funnelshift_r(w[i], w[(i + 1) % NW], sh);
#pragma unroll
            for (int k = 0; k < 8; ++k)
              nib_step<NH4, Lo::HALF_I, PDI * 16>(accI, R, k, lb, 8 * i + k);
          }
        } else {
          // 64 index bytes (two 3-bit codes in nibbles), rotated by `lane` bytes
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
              const int s = 4 * i + k;
              const uint32_t v = (R >> (8 * k)) & 0xffu;
              const int msk = static_cast<int>(v << 25) >> 31;          // bit 6: high code >= 4
              const uint32_t vc = v ^ (static_cast<uint32_t>(msk) & 0x77u);
              const uint32_t en = (vc & 7u) | ((vc >> 1) & 0x18u);
              const uint32_t p6 = static_cast<uint32_t>((lane + s) & 63);
              lut_acc<NH4, Lo::HALF_I>(accI, lutI + (en * PDI + p6) * 16, sign_pair(msk));
            }
          }
        }
        const uint32_t nn = reinterpret_cast<const uint32_t*>(cur + Lo::o_nrm)[my];
        const float n16 = half_lo(nn), r16 = half_hi(nn);
        float sc[NH];
#pragma unroll
        for (int j = 0; j < NH / 2; ++j) {
          const float2 xi = up2(accI[j]), xs = up2(accS[j]);
          sc[2 * j] = fmaf(n16, xi.x, r16 * xs.x);
          sc[2 * j + 1] = fmaf(n16, xi.y, r16 * xs.y);
        }
        if (a.scores != nullptr && valid) {
#pragma unroll
          for (int h = 0; h < NH; ++h) {
            if (h < nh) {
              const int hq = a.g_heads[grp][h];
              a.scores[(static_cast<int64_t>(b) * a.n_q_heads + hq) * a.scores_ld + ts + my] =
                  sc[h] * a.inv_scale_log2;
            }
          }
        }
        if constexpr (HAS_V) {
          // online softmax (b3): p pairs and this token's dequant pairs to shared
          float p[NH];
#pragma unroll
          for (int h = 0; h < NH; ++h) {
            const float s = (valid && h < nh) ? sc[h] : -INFINITY;
            const float mx = warp_max(s);
            const float mn = fmaxf(m[h], mx);
            const float alpha = mn == -INFINITY ? 1.f : exp2f(m[h] - mn);
            p[h] = mn == -INFINITY ? 0.f : exp2f(s - mn);
            l[h] = fmaf(l[h], alpha, p[h]);
            const uint64_t al = pk2(alpha, alpha);
            o[h][0] = mul2(o[h][0], al);
            o[h][1] = mul2(o[h][1], al);
            m[h] = mn;
          }
          uint64_t* myp = sPP + lane * kMaxHeads;
#pragma unroll
          for (int h = 0; h < NH; h += 2)
            *reinterpret_cast<ulonglong2*>(myp + h) = make_ulonglong2(pk2(p[h], p[h]), pk2(p[h + 1], p[h + 1]));
          {
            // v_hat = mn16 + code * s16 = f * (16 s16) + (mn16 - 16 s16), f = 1 + code / 16
            const uint4 par = *reinterpret_cast<const uint4*>(cur + Lo::o_vp + my * 16);
            const uint32_t pw[4] = {par.x, par.y, par.z, par.w};
#pragma unroll
            for (int g = 0; g < 4; ++g) {
              const float mnv = half_lo(pw[g]), scv = half_hi(pw[g]);
              const float s16 = 16.f * scv, cc = fmaf(-16.f, scv, mnv);
              sVP[lane * 4 + g] = make_float4(s16, s16, cc, cc);
            }
          }
          __syncwarp();

          // P.V (b4): lane owns channels 4 lane .. 4 lane + 3 (group lane / 8), one token a step
          const int vg = lane >> 3;
#pragma unroll 2
          for (int i = 0; i < wcount; ++i) {
            const int tok = 32 * warp + i;
            const float4 dq = sVP[i * 4 + vg];
            const uint64_t S16 = pk2(dq.x, dq.y), CC = pk2(dq.z, dq.w);
            uint32_t c0, c1, c2, c3;
            if constexpr (VB == 2) {
              const uint32_t by = cur[Lo::o_vq + tok * 32 + lane];
              c0 = by << 19; c1 = by << 17; c2 = by << 15; c3 = by << 13;
              c0 &= 0x00180000u; c1 &= 0x00180000u; c2 &= 0x00180000u; c3 &= 0x00180000u;
            } else {
              const uint32_t hw = reinterpret_cast<const uint16_t*>(cur + Lo::o_vq + tok * 64)[lane];
              c0 = (hw << 19) & 0x00780000u; c1 = (hw << 15) & 0x00780000u;
              c2 = (hw << 11) & 0x00780000u; c3 = (hw << 7) & 0x00780000u;
            }
            const uint64_t f01 = pk2(__uint_as_float(0x3f800000u | c0), __uint_as_float(0x3f800000u | c1));
            const uint64_t f23 = pk2(__uint_as_float(0x3f800000u | c2), __uint_as_float(0x3f800000u | c3));
            const uint64_t v01 = fma2(f01, S16, CC), v23 = fma2(f23, S16, CC);
            const uint64_t* pp = sPP + i * kMaxHeads;
#pragma unroll
            for (int h = 0; h < NH; h += 2) {
              const ulonglong2 ph = *reinterpret_cast<const ulonglong2*>(pp + h);
              o[h][0] = fma2(ph.x, v01, o[h][0]);
              o[h][1] = fma2(ph.x, v23, o[h][1]);
              o[h + 1][0] = fma2(ph.y, v01, o[h + 1][0]);
              o[h + 1][1] = fma2(ph.y, v23, o[h + 1][1]);
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

  // ---------------- merge the 8 warps of this CTA (b5)
  __syncthreads();
  float* sM = reinterpret_cast<float*>(tiles);  // [warp][head][kPartStride]
#pragma unroll
  for (int h = 0; h < NH; ++h) {
    if (h < nh) {
      const float lt = warp_sum(l[h]);
      float* dst = sM + (warp * kMaxHeads + h) * kPartStride;
      if (lane == 0) { dst[0] = m[h]; dst[1] = lt; }
      const float2 v0 = up2(o[h][0]), v1 = up2(o[h][1]);
      *reinterpret_cast<float4*>(dst + 4 + 4 * lane) = make_float4(v0.x, v0.y, v1.x, v1.y);
    }
  }
  __syncthreads();
  if (warp < nh) {
    const int h = warp, hq = a.g_heads[grp][h];
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < 8; ++w) M = fmaxf(M, sM[(w * kMaxHeads + h) * kPartStride]);
    float Lsum = 0.f, O[4] = {0.f, 0.f, 0.f, 0.f};
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < 8; ++w) {
        const float* src = sM + (w * kMaxHeads + h) * kPartStride;
        if (src[0] == -INFINITY) continue;
        const float f = exp2f(src[0] - M);
        Lsum = fmaf(f, src[1], Lsum);
        const float4 ov = *reinterpret_cast<const float4*>(src + 4 + 4 * lane);
        O[0] = fmaf(f, ov.x, O[0]);
        O[1] = fmaf(f, ov.y, O[1]);
        O[2] = fmaf(f, ov.z, O[2]);
        O[3] = fmaf(f, ov.w, O[3]);
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

  // ---------------- the last CTA of this (sequence, head group) merges all splits
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    int* ctr = a.counters + static_cast<int64_t>(b) * a.n_q_heads + a.g_heads[grp][0];
    sLast = atomicAdd(ctr, 1) == a.n_splits - 1;
  }
  __syncthreads();
  if (!sLast) return;
  __threadfence();
  // one warp per head, heads in parallel: lanes read the split maxima and sums (lane = split),
  // then the weighted partial outputs are loaded 16 splits at a time (independent loads)
  if (warp < nh) {
    const int h = warp, hq = a.g_heads[grp][h];
    const float* base = a.part + (static_cast<int64_t>(b) * a.n_q_heads + hq) * a.n_splits * kPartStride;
    float mloc = -INFINITY;
    for (int s = lane; s < a.n_splits; s += 32) mloc = fmaxf(mloc, __ldcg(base + s * kPartStride));
    const float M = warp_max(mloc);
    float Lsum = 0.f, O[4] = {0.f, 0.f, 0.f, 0.f};
    if (M != -INFINITY) {
      for (int s0 = 0; s0 < a.n_splits; s0 += 32) {
        const int s = s0 + lane;
        float f = 0.f;
        if (s < a.n_splits) {
          const float ms = __ldcg(base + s * kPartStride);
          const float lsv = __ldcg(base + s * kPartStride + 1);
          if (ms != -INFINITY) {
            f = exp2f(ms - M);
            Lsum = fmaf(f, lsv, Lsum);
          }
        }
        const int cnt = min(32, a.n_splits - s0);
        const float* blk = base + s0 * kPartStride + 4 + 4 * lane;
        int j = 0;
        for (; j + 16 <= cnt; j += 16) {
          float4 ov[16];
#pragma unroll
          for (int u = 0; u < 16; ++u) ov[u] = __ldcg(reinterpret_cast<const float4*>(blk + (j + u) * kPartStride));
#pragma unroll
          for (int u = 0; u < 16; ++u) {
            const float fj = __shfl_sync(kFull, f, j + u);
            O[0] = fmaf(fj, ov[u].x, O[0]);
            O[1] = fmaf(fj, ov[u].y, O[1]);
            O[2] = fmaf(fj, ov[u].z, O[2]);
            O[3] = fmaf(fj, ov[u].w, O[3]);
          }
        }
        for (; j < cnt; ++j) {
          const float fj = __shfl_sync(kFull, f, j);
          const float4 ov = __ldcg(reinterpret_cast<const float4*>(blk + j * kPartStride));
          O[0] = fmaf(fj, ov.x, O[0]);
          O[1] = fmaf(fj, ov.y, O[1]);
          O[2] = fmaf(fj, ov.z, O[2]);
          O[3] = fmaf(fj, ov.w, O[3]);
        }
      }
      Lsum = warp_sum(Lsum);
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

template <int MB, int VB, int NH4>
tq_status run_decode(const DecodeArgs& a, dim3 grid, cudaStream_t st) {
  constexpr int smem = Lay<MB, VB, NH4>::total;
  static_assert(smem <= 227 * 1024, "decode shared memory budget");
  auto kern = k_decode<MB, VB, NH4>;
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

template <int MB, int VB>
tq_status run_decode_nh(const DecodeArgs& a, dim3 grid, int max_heads, cudaStream_t st) {
  return max_heads <= 4 ? run_decode<MB, VB, 1>(a, grid, st) : run_decode<MB, VB, 2>(a, grid, st);
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

  // head groups: the query heads of each KV head, in balanced groups of at most 8
  int n_groups = 0, max_heads = 0;
  for (int kv = 0; kv < c->n_kv_heads; ++kv) {
    int heads[1024];
    int n = 0;
    for (int h = 0; h < n_q_heads; ++h)
      if ((head_map ? head_map[h] : h / (n_q_heads / c->n_kv_heads)) == kv) heads[n++] = h;
    if (n == 0) continue;
    const int ng = (n + kMaxHeads - 1) / kMaxHeads;
    int pos = 0;
    for (int g = 0; g < ng; ++g) {
      const int cnt = (n - pos) / (ng - g);
      if (n_groups >= kMaxGroups) return TQ_EUNSUPPORTED;
      a.g_kv[n_groups] = static_cast<int16_t>(kv);
      a.g_n[n_groups] = static_cast<int8_t>(cnt);
      for (int i = 0; i < cnt; ++i) a.g_heads[n_groups][i] = static_cast<int16_t>(heads[pos + i]);
      max_heads = cnt > max_heads ? cnt : max_heads;
      pos += cnt;
      ++n_groups;
    }
  }
  if (n_groups == 0) return TQ_OK;

  int max_len = 0;
  for (int b = 0; b < c->batch; ++b) max_len = c->len_host[b] > max_len ? c->len_host[b] : max_len;
  if (max_len == 0 && out == nullptr) return TQ_OK;

  // split count: minimise (CTAs per SM) x (tokens per split + per-CTA set-up) + the final
  // combine; CTAs sharing an SM share its issue slots, so they count as serial work
  int dev = 0;
  cudaGetDevice(&dev);
  const int sms = sm_count(dev);
  const int pairs = c->batch * n_groups;
  const int cap_splits = max_splits_for(c->capacity);
  int best = 1;
  double best_cost = 1e300;
  const int max_try = std::max(1, std::min(cap_splits, (max_len + 127) / 128));
  for (int s = 1; s <= max_try; ++s) {
    const int tps = ((max_len + s - 1) / s + 31) & ~31;
    const int used = (max_len + tps - 1) / tps;
    if (used != s) continue;
    const double waves = std::ceil(static_cast<double>(pairs) * s / sms);
    const double cost = waves * (tps + 256.0) + (s > 1 ? 4.0 * s : 0.0);
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
    case 1 * 8 + 0: return run_decode_nh<1, 0>(a, grid, max_heads, st);
    case 1 * 8 + 2: return run_decode_nh<1, 2>(a, grid, max_heads, st);
    case 1 * 8 + 4: return run_decode_nh<1, 4>(a, grid, max_heads, st);
    case 2 * 8 + 0: return run_decode_nh<2, 0>(a, grid, max_heads, st);
    case 2 * 8 + 2: return run_decode_nh<2, 2>(a, grid, max_heads, st);
    case 2 * 8 + 4: return run_decode_nh<2, 4>(a, grid, max_heads, st);
    case 3 * 8 + 0: return run_decode_nh<3, 0>(a, grid, max_heads, st);
    case 3 * 8 + 2: return run_decode_nh<3, 2>(a, grid, max_heads, st);
    case 3 * 8 + 4: return run_decode_nh<3, 4>(a, grid, max_heads, st);
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
