// Fused decode attention over a packed KV cache: prod, mse or grouped keys (sm_100a).
//
// Estimator (Implementing TurboQuant (part 5), algorithm overview; validate_paper.py
// attention_score):  s_i = n16_i <Pi q, c[idx_i]> + r16_i sqrt(pi/2)/d <S q, 2 sigma_i - 1>.
// With q_rot = H (s . q) (so Pi q = q_rot / sqrt(d)) and Sq = S_rot q_rot / sqrt(d):
//   <Pi q, c[idx]> = (1/d) sum_j q_rot_j C[idx_j]      (C: N(0,1)-scale centroids).
// Both sums are read from per-query byte lookup tables in shared memory; the kernel consumes
// the packed bytes directly (TurboQuant bit-packing article, section 5).
//
// Byte tables. Every packed byte is one lookup: a 2-bit index byte covers 4 coordinates, a
// 1-bit index byte 8, a byte of two 3-bit indices (in nibbles) 2, a QJL sign byte 8. The
// Lloyd-Max codebook is symmetric (C[L-1-k] = -C[k]) and the sign sums are odd, so the value
// of a byte and of its mirror (every code k -> L-1-k, every sign flipped) differ only in sign:
// a table keeps the canonical half (top bit clear) and a lookup returns (entry, +-1). An
// entry holds 4 query heads (16 bytes); a CTA serves at most 4 heads. Entry e of position p
// sits at (e * P + p) * 16 bytes. At step i of an 8-position block, lane l reads position
// 8 b + ((l + i) mod 8), so the eight lanes of one 16-byte shared-memory phase fall in eight
// different bank groups. Tables are pre-multiplied by sm_scale * log2(e): the online softmax
// runs in base 2.
//
// Grid: (context split, head group, sequence); a CTA takes one KV head, up to 4 of its query
// heads and a contiguous token range, with 16 warps. Warp w walks its own 32-token chunks
// (chunk w, w + 16, ... of the range), so no CTA-wide barrier sits in the loop: each lane
// holds its token's key bytes in registers (prefetched one chunk ahead), scores it from the
// tables, and the warp runs the online softmax; the chunk's value bytes arrive in the warp's
// own shared-memory slot by cp.async, and for P.V each half-warp takes one token a step with
// its 16 lanes splitting the 128 channels (8 per lane) in packed fp32x2 FMAs. Each CTA merges
// its warps and writes a partial (m, l, o); the last CTA of a (sequence, head group) to finish
// merges all partials (an atomic counter, no waiting), or writes the merged partial itself
// for a context-parallel decode.
#include <atomic>
#include <cfloat>
#include <cmath>
#include <mutex>

#include "tq_device.cuh"
#include "tq_internal.h"

namespace tq {
namespace {

constexpr int kMaxHeads = 4;      // query heads of one table set (one 16-byte table entry)
constexpr int kMaxSlots = 8;      // query heads per CTA: at most two table sets
constexpr int kMaxGroups = 256;
std::atomic<int> g_decode_policy{TQ_DECODE_AUTO};
constexpr int kPartStride = 132;  // floats per (head, split) partial: m, l, pad, o[128]
constexpr int kSrotStride = 272;  // bytes per staged q half row (256 + 16: bank spread)
// dequant pairs of a warp: [group][token] float4 rows of 34 entries, so that the 4 groups x 2
// tokens read by one P.V step fall in 8 different 16-byte bank groups
constexpr int kVpStride = 34;

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
  float* part_out;  // nullable: per (sequence, query head) (m, l, o) records instead of out
  float* part;
  int* counters;
  const DevTables* tab;
  int64_t scores_ld;
  int n_kv_heads, capacity, n_q_heads;
  int q_f32, out_f32;
  int n_splits, tokens_per_split;
  int max_len;  // host copy of the longest sequence (an upper bound of every len[b])
  float scale_log2, inv_scale_log2;
  int16_t g_kv[kMaxGroups];
  int16_t g_heads[kMaxGroups][kMaxSlots];
  int8_t g_n[kMaxGroups];
};

// Programmatic dependent launch: wait until the grids this one depends on have completed and
// their memory is visible (a no-op when the kernel was launched without the attribute).
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
}

// (+1.0, +1.0) or (-1.0, -1.0) from an all-ones / all-zeros mask
__device__ __forceinline__ uint64_t sign_pair(int mask) {
  const float s = __uint_as_float(0x3f800000u | (static_cast<uint32_t>(mask) & 0x80000000u));
  return pk2(s, s);
}

// Key kinds: mse (indices, one norm), prod (indices + QJL signs, two norms), grouped (a
// 32-channel outlier group at b + 1 bits and a 96-channel group at b bits, one norm each).
enum KeyKind { kMse = 0, kProd = 1, kGrp = 2 };

// CTA shape for NSET table sets of 4 head slots: 16 warps with one set, 12 with two (whose
// tables and per-head state take more of the shared memory and registers).
template <int NSET>
struct Cfg {
  static constexpr int slots = kMaxHeads * NSET;            // head slots
  static constexpr int threads = NSET == 1 ? 512 : 384;
  static constexpr int warps = threads / 32;
  static constexpr int chunk_stride = 32 * warps;           // tokens between a warp's chunks
};

// Shared-memory plan. MB: index bits (mse, prod) or the grouped base bits b. A token's key
// bytes form two lookup segments: I (index bytes; grouped: the outlier group) and S (prod:
// the QJL sign bytes; grouped: the normal group, padded with zero bytes to whole 8-byte
// blocks). Each segment accumulates its own sum; the two norms scale them.
template <int MB, int VB, int K, int NSET, bool NIBT = false>
struct Lay {
  static constexpr int SL = Cfg<NSET>::slots, kWarps = Cfg<NSET>::warps;
  static constexpr bool GRP = K == kGrp;
  static constexpr int MI = GRP ? MB + 1 : MB;                     // segment I code bits
  static constexpr int MS = GRP ? MB : 1;                          // segment S code bits
  static constexpr int IBI = (GRP ? 32 : kD) * storage_width_c(MI) / 8;
  static constexpr int IBS = GRP ? 96 * storage_width_c(MS) / 8 : 0;
  static constexpr int IB = IBI + IBS;                             // index-plane bytes per token
  static constexpr int PI = IBI;                                   // segment I positions
  static constexpr int EI = MI == 3 ? 32 : 128;                    // canonical entries per position
  static constexpr int PS = K == kProd ? 16 : (GRP ? (IBS + 7) / 8 * 8 : 0);
  static constexpr int ES = MS == 3 ? 32 : 128;
  static constexpr int KW = (IBI + (GRP ? PS : 0)) / 4;            // key words held per token
  static constexpr int NB = K == kMse ? 2 : 4;                     // norm bytes per token
  static constexpr int VQB = VB ? kD * VB / 8 : 0;         // value code bytes per token
  static constexpr int VPB = VB ? 16 : 0;                  // value params per token
  // Tables: NSET sets (head slots 4s .. 4s + 3), each set contiguous. NIBT: the QJL sign
  // tables are nibble tables (16 entries x 32 nibble positions, no mirror), which keeps two
  // sets of 3-bit prod tables within the shared memory.
  static constexpr bool NIB = NIBT;
  static constexpr int SETI = EI * PI * 16;                          // bytes of one index set
  static constexpr int SETS = NIB ? 16 * 32 * 16 : ES * PS * 16;     // bytes of one sign set
  static constexpr int lutI = 0;
  static constexpr int lutS = lutI + NSET * SETI;
  static constexpr int qrT = lutS + NSET * SETS;                     // q_rot [128][SL] f32
  static constexpr int sqT = qrT + kD * SL * 4;               // Sq    [128][SL] f32
  static constexpr int qhi = sqT + kD * SL * 4;               // hi [8][136] f16
  static constexpr int qlo = qhi + 8 * kSrotStride;                  // lo [8][136] f16
  static constexpr int qinv = qlo + 8 * kSrotStride;                 // [8] f32
  // per-warp slots: value bytes of the chunk, p pairs, dequant pairs
  static constexpr int wv = (qinv + 32 + 127) & ~127;
  static constexpr int wv_bytes = 32 * (VQB + VPB);
  static constexpr int o_vq = 0;                 // within a warp's value slot
  static constexpr int o_vp = 32 * VQB;
  static_assert(o_vq == 0 && o_vp >= 0, "value slot layout");
  static constexpr int ppair = wv + kWarps * wv_bytes;                 // [warp][32][SL] (p, p) pairs
  static constexpr int vpair = ppair + kWarps * 32 * SL * 8;    // [warp][4][34] f32x4
  static constexpr int end_v = vpair + (VB ? kWarps * 4 * kVpStride * 16 : 0);
  static constexpr int merge = kWarps * SL * kPartStride * 4;   // reuses wv..
  // prologue scratch for the nibble partial tables (the value slots may be filling then)
  static constexpr int PNI = MI == 3 ? 0 : PI;                         // nibble-built positions
  static constexpr int PNS = MS == 3 ? 0 : PS;
  static constexpr int scratch = VB ? ppair : wv;
  static constexpr int scratch_bytes = NSET * (2 * 16 * PNI + (NIB ? 0 : 2 * 16 * PNS)) * 16;
  // the last CTA's merge: split maxima, sums and weights per head slot, 4 SL floats, and
  // (slice, active head) partial sums (at most one slice of 32 float4 per warp)
  static constexpr int last = 3 * SL * 256 * 4 + 4 * SL * 4 + kWarps * 32 * 16;
  static constexpr int need_wv = merge > last ? merge : last;
  static constexpr int total0 = (end_v - wv) >= need_wv ? end_v : wv + need_wv;
  static constexpr int total = total0 >= scratch + scratch_bytes ? total0 : scratch + scratch_bytes;
  static_assert(IBI % 8 == 0 && PS % 8 == 0, "whole 8-byte lookup blocks");
  static_assert(NSET == 1 || K != kGrp, "grouped keys use one table set");
  static constexpr bool fits = total <= 227 * 1024;                  // decode shared memory budget
};

// The layout a kernel uses: byte sign tables (16 lookups a key) where they fit, else nibble
// sign tables (32 lookups a key, 4 times smaller) for two sets of prod tables.
template <int MB, int VB, int K, int NSET>
struct LayPick {
  static constexpr bool nib = K == kProd && NSET == 2 && !Lay<MB, VB, K, NSET, false>::fits;
  using type = Lay<MB, VB, K, NSET, nib>;
};

// Accumulate one 4-head table entry of each of the NS table sets (SETB bytes apart) with
// sign: acc[s][j] += sg * entry_s.
template <int NS, int SETB>
__device__ __forceinline__ void lut_acc(uint64_t (&acc)[NS][2], const uint8_t* p, uint64_t sg) {
#pragma unroll
  for (int s = 0; s < NS; ++s) {
    const ulonglong2 L = *reinterpret_cast<const ulonglong2*>(p + s * SETB);
    acc[s][0] = fma2(sg, L.x, acc[s][0]);
    acc[s][1] = fma2(sg, L.y, acc[s][1]);
  }
}

// Byte k of w sign-extended to 32 bits (prmt: a selector nibble with its top bit set
// replicates the selected byte's sign bit).
__device__ __forceinline__ int byte_sx(uint32_t w, int k) {
  const uint32_t sel = static_cast<uint32_t>(k) | ((8u | k) << 4) | ((8u | k) << 8) | ((8u | k) << 12);
  uint32_t d;
  asm("prmt.b32 %0, %1, 0, %2;" : "=r"(d) : "r"(w), "r"(sel));
  return static_cast<int>(d);
}

// The 8-byte block (w0, w1) rotated right by this lane's r = l mod 8 bytes: byte i of
// (out0, out1) is byte (r + i) mod 8 of the block.
__device__ __forceinline__ void rot_block(uint32_t w0, uint32_t w1, bool swap, uint32_t sh,
                                          uint32_t& out0, uint32_t& out1) {
  const uint32_t a = swap ? w1 : w0, b = swap ? w0 : w1;
  out0 = __funnelshift_r(a, b, sh);
  out1 = __funnelshift_r(b, a, sh);
}

// Lookups of one 8-byte block of mirror-symmetric bytes (index bytes of 1-, 2- or 4-bit
// codes, or sign bytes): byte i of the rotated block is position 8 blk + ((l + i) mod 8).
template <int ROWB, int NS, int SETB>
__device__ __forceinline__ void block_lookups(uint64_t (&acc)[NS][2], uint32_t R0, uint32_t R1,
                                              const uint8_t* tab, int blk,
                                              const uint32_t (&rot16)[8]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t R = i < 4 ? R0 : R1;
    const int sx = byte_sx(R, i & 3);
    const int msk = sx >> 31;
    const uint32_t e = static_cast<uint32_t>(sx ^ msk);  // canonical entry, 0..127
    lut_acc<NS, SETB>(acc, tab + 128 * blk + e * ROWB + rot16[i], sign_pair(msk));
  }
}

// Lookups of one 8-byte block of bytes holding two 3-bit codes in their nibbles: the mirror
// flips both codes (k -> 7 - k), chosen by bit 6 (high code >= 4); entry = low code + 8 (high
// code mod 4).
template <int ROWB, int NS, int SETB>
__device__ __forceinline__ void block_lookups3(uint64_t (&acc)[NS][2], uint32_t R0, uint32_t R1,
                                               const uint8_t* tab, int blk,
                                               const uint32_t (&rot16)[8]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t v = ((i < 4 ? R0 : R1) >> (8 * (i & 3))) & 0xffu;
    const int msk = static_cast<int>(v << 25) >> 31;
    const uint32_t vc = v ^ (static_cast<uint32_t>(msk) & 0x77u);
    const uint32_t en = (vc & 7u) | ((vc >> 1) & 0x18u);
    lut_acc<NS, SETB>(acc, tab + 128 * blk + en * ROWB + rot16[i], sign_pair(msk));
  }
}

// Segment lookups over 8-byte blocks of words w (2 words a block).
template <int MBITS, int NPOS, int NS, int SETB>
__device__ __forceinline__ void segment_lookups(uint64_t (&acc)[NS][2], const uint32_t* w,
                                                const uint8_t* tab, bool swap, uint32_t sh,
                                                const uint32_t (&rot16)[8]) {
#pragma unroll
  for (int blk = 0; blk < NPOS / 8; ++blk) {
    uint32_t R0, R1;
    rot_block(w[2 * blk], w[2 * blk + 1], swap, sh, R0, R1);
    if constexpr (MBITS == 3) block_lookups3<NPOS * 16, NS, SETB>(acc, R0, R1, tab, blk, rot16);
    else block_lookups<NPOS * 16, NS, SETB>(acc, R0, R1, tab, blk, rot16);
  }
}

// QJL sign lookups from nibble tables (16 entries x 32 nibble positions, entry e of position
// p at (e 32 + p) 16 bytes): the 128 sign bits as 32 nibbles. Each 32-bit word (8 nibble
// positions) is rotated by this lane's 4 (l mod 8) bits, so that at step i lane l reads
// position 8 blk + ((l + i) mod 8) and the eight lanes of a 16-byte phase fall in eight
// different bank groups.
template <int NS, int SETB>
__device__ __forceinline__ void nibble_lookups(uint64_t (&acc)[NS][2], const uint32_t (&w)[4],
                                               const uint8_t* tab, uint32_t r8,
                                               const uint32_t (&rot16)[8]) {
#pragma unroll
  for (int blk = 0; blk < 4; ++blk) {
    const uint32_t rot = __funnelshift_r(w[blk], w[blk], 4 * r8);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint8_t* p = tab + ((rot >> (4 * i)) & 15u) * 512 + blk * 128 + rot16[i];
#pragma unroll
      for (int s = 0; s < NS; ++s) {
        const ulonglong2 L = *reinterpret_cast<const ulonglong2*>(p + s * SETB);
        acc[s][0] = add2(acc[s][0], L.x);
        acc[s][1] = add2(acc[s][1], L.y);
      }
    }
  }
}

// K = kMse: s = n16 <Pi q, c[idx]>; kProd: + r16 sqrt(pi/2)/d <S q, 2 sigma - 1>;
// kGrp: s = n_o <Pi_o q_o, c_o[idx_o]> + n_n <Pi_n q_n, c_n[idx_n]> over the two channel
// groups (Pi_g: 32-point Hadamard blocks after the group's signs).
template <int MB, int VB, int NH, int K, int NSET>
__global__ void __launch_bounds__(Cfg<NSET>::threads, 1) k_decode(const __grid_constant__ DecodeArgs a) {
  using Lo = typename LayPick<MB, VB, K, NSET>::type;
  constexpr int NT = Cfg<NSET>::threads, NWp = Cfg<NSET>::warps, CS = Cfg<NSET>::chunk_stride;
  constexpr int SL = Cfg<NSET>::slots;
  constexpr bool PROD = K == kProd, GRP = K == kGrp, TWO = K != kMse;
  constexpr int IB = Lo::IB, PI = Lo::PI, KW = Lo::KW;
  static_assert(NH >= 1 && NH <= SL, "heads per CTA");
  static_assert(Lo::fits, "decode shared memory budget");
  constexpr bool HAS_V = VB != 0;
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* lutI = smem + Lo::lutI;
  uint8_t* lutS = smem + Lo::lutS;
  float* qrT = reinterpret_cast<float*>(smem + Lo::qrT);
  float* sqT = reinterpret_cast<float*>(smem + Lo::sqT);
  uint8_t* qhi = smem + Lo::qhi;
  uint8_t* qlo = smem + Lo::qlo;
  float* qinv = reinterpret_cast<float*>(smem + Lo::qinv);
  __shared__ int sLast;
  __shared__ float sCen[32];

  const int split = blockIdx.x, grp = blockIdx.y, b = blockIdx.z;
  const int kv = a.g_kv[grp], nh = a.g_n[grp];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int t0 = split * a.tokens_per_split;
  const int64_t kvrow = (static_cast<int64_t>(b) * a.n_kv_heads + kv) * a.capacity;

  // P.V, one table set: half-warp hw = lane / 16 takes every other token of a chunk and lane
  // owns channels 8 j16 .. 8 j16 + 7 (j16 = lane mod 16) as four fp32 pairs; two sets (up to 8
  // heads, whose accumulators would not fit twice): the warp takes one token a step and lane
  // owns channels 4 lane .. 4 lane + 3 as two pairs.
  constexpr int OC = NSET == 1 ? 4 : 2;
  float m[NH], l[NH];
  uint64_t o[NH][OC];
#pragma unroll
  for (int h = 0; h < NH; ++h) {
    m[h] = -INFINITY;
    l[h] = 0.f;
#pragma unroll
    for (int k = 0; k < OC; ++k) o[h][k] = 0ull;
  }

  // The prologue reads only the query and the quantizer's tables, so it runs before the
  // grid-dependency wait: launched after tq_append, it overlaps the append kernel (which
  // signals its dependents at entry). The lengths and the cache are read after the wait.
  int t1 = t0;
  if (t0 < a.max_len) {
    // warm L2 with this CTA's packed rows (all of them lie below the capacity); the reads
    // proper come after the dependency wait (L2 is the point of coherence for the append)
    {
      const int tp1 = min(a.max_len, t0 + a.tokens_per_split);
      const int n = tp1 - t0;
      const uint8_t* rng[5] = {a.k_idx + (kvrow + t0) * IB, a.k_sgn + (kvrow + t0) * 16,
                               reinterpret_cast<const uint8_t*>(a.k_nrm) + (kvrow + t0) * Lo::NB,
                               a.v_q + (kvrow + t0) * Lo::VQB,
                               reinterpret_cast<const uint8_t*>(a.v_par) + (kvrow + t0) * 16};
      const int len_b[5] = {n * IB, PROD ? n * 16 : 0, n * Lo::NB, n * Lo::VQB, VB ? n * 16 : 0};
#pragma unroll
      for (int r = 0; r < 5; ++r)
        for (int off = threadIdx.x * 128; off < len_b[r]; off += NT * 128)
          asm volatile("prefetch.global.L2 [%0];" ::"l"(rng[r] + off));
    }
    // key bytes of this lane's token in chunk c (zeros past the range)
    // (grouped: the normal group's words are zero-padded to whole 8-byte blocks)
    uint32_t kw[KW], sw4[4], nw;
    auto load_keys = [&](int ts, uint32_t (&iw)[KW], uint32_t (&sg)[4], uint32_t& nn) {
      const int t = ts + lane;
#pragma unroll
      for (int i = IB / 4; i < KW; ++i) iw[i] = 0u;
      if (t < t1) {
        const uint8_t* row = a.k_idx + (kvrow + t) * IB;
        if constexpr (IB % 16 == 0) {
#pragma unroll
          for (int i = 0; i < IB / 16; ++i) {
            const uint4 v = __ldg(reinterpret_cast<const uint4*>(row) + i);
            iw[4 * i] = v.x; iw[4 * i + 1] = v.y; iw[4 * i + 2] = v.z; iw[4 * i + 3] = v.w;
          }
        } else if constexpr (IB % 8 == 0) {
#pragma unroll
          for (int i = 0; i < IB / 8; ++i) {
            const uint2 v = __ldg(reinterpret_cast<const uint2*>(row) + i);
            iw[2 * i] = v.x; iw[2 * i + 1] = v.y;
          }
        } else {
#pragma unroll
          for (int i = 0; i < IB / 4; ++i) iw[i] = __ldg(reinterpret_cast<const uint32_t*>(row) + i);
        }
        if constexpr (PROD) {
          const uint4 s4 = __ldg(reinterpret_cast<const uint4*>(a.k_sgn + (kvrow + t) * 16));
          sg[0] = s4.x; sg[1] = s4.y; sg[2] = s4.z; sg[3] = s4.w;
        } else {
          sg[0] = sg[1] = sg[2] = sg[3] = 0u;
        }
        if constexpr (TWO) nn = __ldg(reinterpret_cast<const uint32_t*>(a.k_nrm) + kvrow + t);
        else nn = __ldg(a.k_nrm + kvrow + t);
      } else {
#pragma unroll
        for (int i = 0; i < IB / 4; ++i) iw[i] = 0u;
        sg[0] = sg[1] = sg[2] = sg[3] = 0u;
        nn = 0u;
      }
    };
    // value bytes of chunk ts into this warp's slot (cp.async, 16-byte pieces)
    uint8_t* wslot = smem + Lo::wv + warp * Lo::wv_bytes;
    auto load_values = [&](int ts) {
      if constexpr (HAS_V) {
        const int n = min(32, t1 - ts);  // tokens of the chunk (>= 1)
        const int cq = n * Lo::VQB / 16, cp = n;
        for (int c = lane; c < cq + cp; c += 32) {
          if (c < cq) cp_async16(wslot + Lo::o_vq + 16 * c, a.v_q + (kvrow + ts) * Lo::VQB + 16 * c, true);
          else cp_async16(wslot + Lo::o_vp + 16 * (c - cq),
                          reinterpret_cast<const uint8_t*>(a.v_par) + (kvrow + ts + (c - cq)) * 16, true);
        }
      }
      cp_async_commit();
    };

    // ---------------- prologue: rotate q, project with S_rot, build the tables
    const DevTables* __restrict__ tab = a.tab;
    // S_rot rows [16 warp, 16 warp + 16) as mma.sync A fragments (warps 0..7), from L2
    uint32_t afr[8][4];
    if (PROD && warp < 8) {
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
    if (warp < 8) {
      // q_rot of head slot `warp` (zeros for empty slots): signs, then the 128-point
      // transform with 4 values per lane (2 stages in registers, 5 across lanes)
      float v[4] = {0.f, 0.f, 0.f, 0.f};
      if (warp < nh) {
        const int hq = a.g_heads[grp][warp];
        const int64_t qoff = (static_cast<int64_t>(b) * a.n_q_heads + hq) * kD;
        if constexpr (GRP) {
          // chain order: the outlier channels, then the normal channels
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int c = tab->chan[4 * lane + i];
            v[i] = a.q_f32 ? static_cast<const float*>(a.q)[qoff + c]
                           : __uint_as_float(static_cast<uint32_t>(static_cast<const uint16_t*>(a.q)[qoff + c]) << 16);
          }
        } else {
          if (a.q_f32) load4<true>(static_cast<const float*>(a.q) + qoff, 4 * lane, v);
          else load4<false>(static_cast<const uint16_t*>(a.q) + qoff, 4 * lane, v);
        }
        const uint32_t sw = tab->sign_bits[lane >> 3];
#pragma unroll
        for (int i = 0; i < 4; ++i) v[i] = flip_sign(v[i], sw, (4 * lane + i) & 31);
        // 128-point transform; grouped: 32-point blocks (lanes 8k .. 8k + 7)
        fwht_reg<4>(v);
#pragma unroll
        for (int mm = 1; mm < (GRP ? 8 : 32); mm <<= 1) {
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
        if (warp < SL) qrT[j * SL + warp] = v[i];
        const float sv = v[i] * scl;
        const __half hi = __float2half_rn(sv);
        const __half lo = __float2half_rn(sv - __half2float(hi));
        reinterpret_cast<__half*>(qhi + warp * kSrotStride)[j] = hi;
        reinterpret_cast<__half*>(qlo + warp * kSrotStride)[j] = lo;
      }
    }
    if (threadIdx.x < 32) sCen[threadIdx.x] = (&tab->cent[0][0])[threadIdx.x];
    __syncthreads();
    if (PROD && warp < 8) {
      // Sq = S_rot q_rot / sqrt(d) for the head slots on tensor cores: mma.sync m16n8k16
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
      if (2 * t < SL) {  // columns 2t, 2t + 1 are head slots
        const float s0 = qinv[2 * t] * 0.088388347648318440550f;      // / sqrt(128)
        const float s1 = qinv[2 * t + 1] * 0.088388347648318440550f;
        const int j0 = 16 * warp + g;
        sqT[j0 * SL + 2 * t] = c0 * s0;
        sqT[j0 * SL + 2 * t + 1] = c1 * s1;
        sqT[(j0 + 8) * SL + 2 * t] = c2 * s0;
        sqT[(j0 + 8) * SL + 2 * t + 1] = c3 * s1;
      }
    }
    __syncthreads();
    // the lookup tables too depend only on the query and the quantizer: built before the
    // grid-dependency wait, they overlap a preceding append as well
    {
      constexpr int PNI = Lo::PNI, PNS = Lo::PNS, PS = Lo::PS;
      const float* cenI = sCen;        // segment I centroids (grouped: the outlier group)
      const float* cenS = sCen + 16;   // grouped: the normal group
      // entry scales: 1/sqrt(d) of Pi times 1/sqrt(d) of the N(0,1)-scale centroids (grouped:
      // 1/sqrt(32) of a Hadamard block times 1/sqrt(d_g)); prod signs: sqrt(pi/2)/d
      const float cI = a.scale_log2 * (GRP ? 1.f / 32.f : 1.f / 128.f);
      const float cS = GRP ? a.scale_log2 * 0.018042195912175807f
                           : a.scale_log2 * 1.2533141373155002512f / 128.f;
      // Entries of 1-, 2- and 4-bit code bytes and of sign bytes are sums of two nibble
      // partials (low and high half of the byte): NI[half][n][p] and NS[half][n][p]
      // (16-byte float4 of a set's 4 head slots) are built in a scratch region first; entry
      // (e, p) = N[0][e mod 16][p] + N[1][e / 16][p]. Table set s holds head slots 4s .. 4s + 3
      // (column 4s of the [128][SL] q_rot and Sq arrays).
      constexpr int NIS = 2 * 16 * PNI, NSS = Lo::NIB ? 0 : 2 * 16 * PNS;  // float4 per set
      float4* NI = reinterpret_cast<float4*>(smem + Lo::scratch);
      float4* NS = NI + NSET * NIS;
#pragma unroll
      for (int st = 0; st < NSET; ++st) {
        if constexpr (PNI > 0) {
          constexpr int CPN = 4 / Lo::MI;  // coordinates per nibble
          for (int i = threadIdx.x; i < NIS; i += NT) {
            const int pp = i % PNI, n = (i / PNI) % 16, hf = i / (16 * PNI);
            float4 r = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int f = 0; f < CPN; ++f) {
              const float4 x = *reinterpret_cast<const float4*>(qrT + (2 * CPN * pp + CPN * hf + f) * SL + 4 * st);
              const float c = cenI[(n >> (Lo::MI * f)) & ((1 << Lo::MI) - 1)] * cI;
              r.x = fmaf(x.x, c, r.x); r.y = fmaf(x.y, c, r.y);
              r.z = fmaf(x.z, c, r.z); r.w = fmaf(x.w, c, r.w);
            }
            NI[st * NIS + (hf * 16 + n) * PNI + pp] = r;
          }
        }
        if constexpr (Lo::NIB) {
          // two sets: QJL sign nibble tables built directly, entry n of nibble position np =
          // sum_f (bit f of n ? +1 : -1) cS Sq_{4 np + f}
          for (int i = threadIdx.x; i < 16 * 32; i += NT) {
            const int np = i % 32, n = i / 32;
            float4 r = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int f = 0; f < 4; ++f) {
              const float4 x = *reinterpret_cast<const float4*>(sqT + (4 * np + f) * SL + 4 * st);
              const float sg = ((n >> f) & 1) ? cS : -cS;
              r.x = fmaf(x.x, sg, r.x); r.y = fmaf(x.y, sg, r.y);
              r.z = fmaf(x.z, sg, r.z); r.w = fmaf(x.w, sg, r.w);
            }
            *reinterpret_cast<float4*>(lutS + st * Lo::SETS + (n * 32 + np) * 16) = r;
          }
        } else if constexpr (PNS > 0) {
          for (int i = threadIdx.x; i < NSS; i += NT) {
            const int pp = i % PNS, n = (i / PNS) % 16, hf = i / (16 * PNS);
            float4 r = make_float4(0.f, 0.f, 0.f, 0.f);
            if constexpr (PROD) {
#pragma unroll
              for (int f = 0; f < 4; ++f) {
                const float4 x = *reinterpret_cast<const float4*>(sqT + (8 * pp + 4 * hf + f) * SL + 4 * st);
                const float sg = ((n >> f) & 1) ? cS : -cS;
                r.x = fmaf(x.x, sg, r.x); r.y = fmaf(x.y, sg, r.y);
                r.z = fmaf(x.z, sg, r.z); r.w = fmaf(x.w, sg, r.w);
              }
            } else if (pp < Lo::IBS) {  // grouped normal group; padding positions stay zero
              constexpr int CPN = 4 / Lo::MS;
#pragma unroll
              for (int f = 0; f < CPN; ++f) {
                const float4 x = *reinterpret_cast<const float4*>(qrT + (32 + 2 * CPN * pp + CPN * hf + f) * SL + 4 * st);
                const float c = cenS[(n >> (Lo::MS * f)) & ((1 << Lo::MS) - 1)] * cS;
                r.x = fmaf(x.x, c, r.x); r.y = fmaf(x.y, c, r.y);
                r.z = fmaf(x.z, c, r.z); r.w = fmaf(x.w, c, r.w);
              }
            }
            NS[st * NSS + (hf * 16 + n) * PNS + pp] = r;
          }
        }
      }
      __syncthreads();
      // bytes of two 3-bit codes in nibbles: coordinates c0 + 2p, c0 + 2p + 1 (entry e: codes
      // e mod 8 and e / 8)
      auto build3 = [&](uint8_t* lut, int P, int c0, const float* cen, float cs, int st) {
        for (int i = threadIdx.x; i < 32 * P; i += NT) {
          const int p = i % P, e = i / P;
          const float4 x = *reinterpret_cast<const float4*>(qrT + (c0 + 2 * p) * SL + 4 * st);
          const float4 y = *reinterpret_cast<const float4*>(qrT + (c0 + 2 * p + 1) * SL + 4 * st);
          const float ca = cen[e & 7] * cs, cb = cen[e >> 3] * cs;
          *reinterpret_cast<float4*>(lut + (e * P + p) * 16) =
              make_float4(fmaf(x.x, ca, y.x * cb), fmaf(x.y, ca, y.y * cb),
                          fmaf(x.z, ca, y.z * cb), fmaf(x.w, ca, y.w * cb));
        }
      };
      auto compose = [&](uint8_t* lut, const float4* N, int P) {
        for (int i = threadIdx.x; i < 128 * P; i += NT) {
          const int pp = i % P, e = i / P;
          const float4 u = N[(e & 15) * P + pp], v = N[(16 + (e >> 4)) * P + pp];
          *reinterpret_cast<float4*>(lut + (e * P + pp) * 16) =
              make_float4(u.x + v.x, u.y + v.y, u.z + v.z, u.w + v.w);
        }
      };
#pragma unroll
      for (int st = 0; st < NSET; ++st) {
        if constexpr (Lo::MI == 3) build3(lutI + st * Lo::SETI, PI, 0, cenI, cI, st);
        else compose(lutI + st * Lo::SETI, NI + st * NIS, PI);
        if constexpr (GRP && Lo::MS == 3) build3(lutS + st * Lo::SETS, PS, 32, cenS, cS, st);
        else if constexpr (PS > 0 && !Lo::NIB) compose(lutS + st * Lo::SETS, NS + st * NSS, PS);
      }
    }
    __syncthreads();
    grid_dependency_wait();
    t1 = min(a.len[b], t0 + a.tokens_per_split);
    const int c0 = t0 + 32 * warp;
    if (c0 < t1) {
      load_keys(c0, kw, sw4, nw);
      load_values(c0);
    }

    // ---------------- main loop: this warp's chunks
    // p pairs of the chunk's tokens: sPP[k 32 + token] = ((p_2k, p_2k), (p_2k+1, p_2k+1))
    ulonglong2* sPP = reinterpret_cast<ulonglong2*>(smem + Lo::ppair) + warp * (SL / 2) * 32;
    float4* sVP = reinterpret_cast<float4*>(smem + Lo::vpair) + warp * 4 * kVpStride;
    const uint32_t r8 = static_cast<uint32_t>(lane & 7);
    const bool swap = r8 >= 4;
    const uint32_t sh = 8 * (r8 & 3);
    uint32_t rot16[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) rot16[i] = ((r8 + i) & 7) * 16;

    for (int ts = c0; ts < t1; ts += CS) {
      // prefetch the next chunk's key bytes
      uint32_t nkw[KW], nsw[4], nnw;
      const int tn = ts + CS;
      if (tn < t1) load_keys(tn, nkw, nsw, nnw);
      const int wcount = min(32, t1 - ts);
      const bool valid = lane < wcount;

      uint64_t accI[NSET][2], accS[NSET][2];
#pragma unroll
      for (int st = 0; st < NSET; ++st) accI[st][0] = accI[st][1] = accS[st][0] = accS[st][1] = 0ull;
      if constexpr (Lo::NIB) nibble_lookups<NSET, Lo::SETS>(accS, sw4, lutS, r8, rot16);
      else if constexpr (PROD) segment_lookups<1, 16, NSET, Lo::SETS>(accS, sw4, lutS, swap, sh, rot16);
      if constexpr (GRP)
        segment_lookups<Lo::MS, Lo::PS, NSET, Lo::SETS>(accS, kw + Lo::IBI / 4, lutS, swap, sh, rot16);
      segment_lookups<Lo::MI, PI, NSET, Lo::SETI>(accI, kw, lutI, swap, sh, rot16);
      const float n16 = half_lo(nw), r16 = TWO ? half_hi(nw) : 0.f;
      float sc[SL];
#pragma unroll
      for (int j = 0; j < SL / 2; ++j) {
        const float2 xi = up2(accI[j / 2][j % 2]), xs = up2(accS[j / 2][j % 2]);
        sc[2 * j] = TWO ? fmaf(n16, xi.x, r16 * xs.x) : n16 * xi.x;
        sc[2 * j + 1] = TWO ? fmaf(n16, xi.y, r16 * xs.y) : n16 * xi.y;
      }
      if (a.scores != nullptr && valid) {
#pragma unroll
        for (int h = 0; h < NH; ++h) {
          if (h < nh) {
            const int hq = a.g_heads[grp][h];
            a.scores[(static_cast<int64_t>(b) * a.n_q_heads + hq) * a.scores_ld + ts + lane] =
                sc[h] * a.inv_scale_log2;
          }
        }
      }
      if constexpr (HAS_V) {
        // online softmax: p pairs and this token's dequant pairs to the warp's slots
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
#pragma unroll
          for (int k = 0; k < OC; ++k) o[h][k] = mul2(o[h][k], al);
          m[h] = mn;
        }
        {
          float pp[SL];  // p of the head slots, zero past NH
#pragma unroll
          for (int h = 0; h < SL; ++h) pp[h] = h < NH ? p[h < NH ? h : 0] : 0.f;
#pragma unroll
          for (int k = 0; k < (NH + 1) / 2; ++k)
            sPP[k * 32 + lane] = make_ulonglong2(pk2(pp[2 * k], pp[2 * k]), pk2(pp[2 * k + 1], pp[2 * k + 1]));
        }
        cp_async_wait<0>();
        __syncwarp();
        {
          // v_hat = mn16 + code * s16 = f * (16 s16) + (mn16 - 16 s16), f = 1 + code / 16
          const uint4 par = *reinterpret_cast<const uint4*>(wslot + Lo::o_vp + lane * 16);
          const uint32_t pw[4] = {par.x, par.y, par.z, par.w};
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            const float mnv = half_lo(pw[g]), scv = half_hi(pw[g]);
            const float s16 = 16.f * scv, cc = fmaf(-16.f, scv, mnv);
            sVP[g * kVpStride + lane] = make_float4(s16, s16, cc, cc);
          }
        }
        __syncwarp();

        if constexpr (NSET == 1) {
          // P.V: token 2 jj + hw of the chunk per step, 8 channels per lane (group j16 / 4)
          const int hw = lane >> 4, j16 = lane & 15, vg = j16 >> 2;
  #pragma unroll 2
          for (int jj = 0; 2 * jj < wcount; ++jj) {
            const int tok = 2 * jj + hw;
            if (tok < wcount) {
              const float4 dq = sVP[vg * kVpStride + tok];
              const uint64_t S16 = pk2(dq.x, dq.y), CC = pk2(dq.z, dq.w);
              uint32_t cw[8];
              if constexpr (VB == 2) {
                const uint32_t c16 = reinterpret_cast<const uint16_t*>(wslot + Lo::o_vq + tok * 32)[j16];
  #pragma unroll
                for (int k = 0; k < 8; ++k) cw[k] = (c16 << (19 - 2 * k)) & 0x00180000u;
              } else {
                const uint32_t c32 = reinterpret_cast<const uint32_t*>(wslot + Lo::o_vq + tok * 64)[j16];
  #pragma unroll
                for (int k = 0; k < 8; ++k)
                  cw[k] = (k < 5 ? (c32 << (19 - 4 * k)) : (c32 >> (4 * k - 19))) & 0x00780000u;
              }
              uint64_t v[4];
  #pragma unroll
              for (int k = 0; k < 4; ++k)
                v[k] = fma2(pk2(__uint_as_float(0x3f800000u | cw[2 * k]), __uint_as_float(0x3f800000u | cw[2 * k + 1])), S16, CC);
              const ulonglong2 p01 = sPP[tok];
  #pragma unroll
              for (int k = 0; k < 4; ++k) {
                o[0][k] = fma2(p01.x, v[k], o[0][k]);
                if constexpr (NH > 1) o[1][k] = fma2(p01.y, v[k], o[1][k]);
              }
              if constexpr (NH > 2) {
                const ulonglong2 p23 = sPP[32 + tok];
  #pragma unroll
                for (int k = 0; k < 4; ++k) {
                  o[2][k] = fma2(p23.x, v[k], o[2][k]);
                  if constexpr (NH > 3) o[3][k] = fma2(p23.y, v[k], o[3][k]);
                }
              }
            }
          }
        } else {
          // P.V: one token of the chunk per step, channels 4 lane .. 4 lane + 3 (group lane / 8)
          const int vg = lane >> 3;
#pragma unroll 2
          for (int tok = 0; tok < wcount; ++tok) {
            const float4 dq = sVP[vg * kVpStride + tok];
            const uint64_t S16 = pk2(dq.x, dq.y), CC = pk2(dq.z, dq.w);
            uint32_t cw[4];
            if constexpr (VB == 2) {
              const uint32_t c8 = wslot[Lo::o_vq + tok * 32 + lane];
#pragma unroll
              for (int k = 0; k < 4; ++k) cw[k] = (c8 << (19 - 2 * k)) & 0x00180000u;
            } else {
              const uint32_t c16 = reinterpret_cast<const uint16_t*>(wslot + Lo::o_vq + tok * 64)[lane];
#pragma unroll
              for (int k = 0; k < 4; ++k) cw[k] = (c16 << (19 - 4 * k)) & 0x00780000u;
            }
            uint64_t v[2];
#pragma unroll
            for (int k = 0; k < 2; ++k)
              v[k] = fma2(pk2(__uint_as_float(0x3f800000u | cw[2 * k]), __uint_as_float(0x3f800000u | cw[2 * k + 1])), S16, CC);
#pragma unroll
            for (int k = 0; k < (NH + 1) / 2; ++k) {
              const ulonglong2 pq = sPP[k * 32 + tok];
              o[2 * k][0] = fma2(pq.x, v[0], o[2 * k][0]);
              o[2 * k][1] = fma2(pq.x, v[1], o[2 * k][1]);
              if (2 * k + 1 < NH) {
                o[(2 * k + 1) % NH][0] = fma2(pq.y, v[0], o[(2 * k + 1) % NH][0]);
                o[(2 * k + 1) % NH][1] = fma2(pq.y, v[1], o[(2 * k + 1) % NH][1]);
              }
            }
          }
        }
        __syncwarp();
        if (tn < t1) load_values(tn);
      }
#pragma unroll
      for (int i = 0; i < KW; ++i) kw[i] = nkw[i];
#pragma unroll
      for (int i = 0; i < 4; ++i) sw4[i] = nsw[i];
      nw = nnw;
    }
    cp_async_wait<0>();
  }
  grid_dependency_wait();  // (CTAs past the longest sequence skipped the wait above)

  if constexpr (!HAS_V) return;

  // ---------------- merge the warps of this CTA
  __syncthreads();
  float* sM = reinterpret_cast<float*>(smem + Lo::wv);  // [warp][head][kPartStride]
#pragma unroll
  for (int h = 0; h < NH; ++h) {
    if constexpr (NSET == 1) {
      // the two half-warps hold disjoint tokens of the same channels
#pragma unroll
      for (int k = 0; k < OC; ++k) {
        const float2 v = up2(o[h][k]);
        o[h][k] = add2(o[h][k], pk2(__shfl_xor_sync(kFull, v.x, 16), __shfl_xor_sync(kFull, v.y, 16)));
      }
    }
    if (h < nh) {
      const float lt = warp_sum(l[h]);
      float* dst = sM + (warp * SL + h) * kPartStride;
      if (lane == 0) { dst[0] = m[h]; dst[1] = lt; }
      if constexpr (NSET == 1) {
        if (lane < 16) {
          const float2 v0 = up2(o[h][0]), v1 = up2(o[h][1]), v2 = up2(o[h][2 % OC]), v3 = up2(o[h][3 % OC]);
          *reinterpret_cast<float4*>(dst + 4 + 8 * lane) = make_float4(v0.x, v0.y, v1.x, v1.y);
          *reinterpret_cast<float4*>(dst + 8 + 8 * lane) = make_float4(v2.x, v2.y, v3.x, v3.y);
        }
      } else {
        const float2 v0 = up2(o[h][0]), v1 = up2(o[h][1]);
        *reinterpret_cast<float4*>(dst + 4 + 4 * lane) = make_float4(v0.x, v0.y, v1.x, v1.y);
      }
    }
  }
  __syncthreads();
  if (warp < nh) {
    const int h = warp, hq = a.g_heads[grp][h];
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NWp; ++w) M = fmaxf(M, sM[(w * SL + h) * kPartStride]);
    float Lsum = 0.f, O[4] = {0.f, 0.f, 0.f, 0.f};
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < NWp; ++w) {
        const float* src = sM + (w * SL + h) * kPartStride;
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
    if (a.n_splits == 1 && a.part_out != nullptr) {
      float* dst = a.part_out + (static_cast<int64_t>(b) * a.n_q_heads + hq) * kPartStride;
      if (lane == 0) *reinterpret_cast<float4*>(dst) = make_float4(M, Lsum, 0.f, 0.f);
      *reinterpret_cast<float4*>(dst + 4 + 4 * lane) = make_float4(O[0], O[1], O[2], O[3]);
    } else if (a.n_splits == 1) {
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
  // Every (head, split) pair's maximum and sum, then every (head, channel quad, split slice)
  // item's weighted partial outputs, are loaded by all threads at once (one round trip each);
  // the slices are summed in shared memory.
  {
    const int S = a.n_splits;
    float* sMx = reinterpret_cast<float*>(smem + Lo::wv);   // [head][S] split maxima
    float* sLs = sMx + SL * 256;                      // [head][S] split sums
    float* sF = sLs + SL * 256;                       // [head][S] weights
    float* sHd = sF + SL * 256;  // [head] 1 / total sum, then [head] maxima and sums
    float4* sAcc = reinterpret_cast<float4*>(sHd + 4 * SL);      // [slice][head][32]
    const float* base = a.part + static_cast<int64_t>(b) * a.n_q_heads * S * kPartStride;
    for (int i = threadIdx.x; i < nh * S; i += NT) {
      const int h = i / S, sp = i - h * S;
      const float* src = base + (static_cast<int64_t>(a.g_heads[grp][h]) * S + sp) * kPartStride;
      sMx[h * 256 + sp] = __ldcg(src);
      sLs[h * 256 + sp] = __ldcg(src + 1);
    }
    __syncthreads();
    if (warp < nh) {
      const int h = warp;
      float mloc = -INFINITY;
      for (int sp = lane; sp < S; sp += 32) mloc = fmaxf(mloc, sMx[h * 256 + sp]);
      const float M = warp_max(mloc);
      float lsum = 0.f;
      for (int sp = lane; sp < S; sp += 32) {
        const float ms = sMx[h * 256 + sp];
        const float f = (M == -INFINITY || ms == -INFINITY) ? 0.f : exp2f(ms - M);
        sF[h * 256 + sp] = f;
        lsum = fmaf(f, sLs[h * 256 + sp], lsum);
      }
      lsum = warp_sum(lsum);
      if (lane == 0) {
        sHd[h] = lsum > 0.f ? 1.f / lsum : 0.f;
        sHd[SL + h] = M;
        sHd[2 * SL + h] = lsum;
      }
    }
    __syncthreads();
    const int G = NT / (32 * nh);  // split slices
    if (threadIdx.x < G * 32 * nh) {
      const int h = threadIdx.x / (32 * G), r = threadIdx.x - h * 32 * G;
      const int qd = r & 31, g = r >> 5;
      const float* src = base + static_cast<int64_t>(a.g_heads[grp][h]) * S * kPartStride + 4 + 4 * qd;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      int sp = g;
      for (; sp + 3 * G < S; sp += 4 * G) {
        float4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) v[u] = __ldcg(reinterpret_cast<const float4*>(src + static_cast<int64_t>(sp + u * G) * kPartStride));
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float f = sF[h * 256 + sp + u * G];
          acc.x = fmaf(f, v[u].x, acc.x); acc.y = fmaf(f, v[u].y, acc.y);
          acc.z = fmaf(f, v[u].z, acc.z); acc.w = fmaf(f, v[u].w, acc.w);
        }
      }
      for (; sp < S; sp += G) {
        const float4 v = __ldcg(reinterpret_cast<const float4*>(src + static_cast<int64_t>(sp) * kPartStride));
        const float f = sF[h * 256 + sp];
        acc.x = fmaf(f, v.x, acc.x); acc.y = fmaf(f, v.y, acc.y);
        acc.z = fmaf(f, v.z, acc.z); acc.w = fmaf(f, v.w, acc.w);
      }
      sAcc[(g * nh + h) * 32 + qd] = acc;
    }
    __syncthreads();
    if (threadIdx.x < 32 * nh) {
      const int h = threadIdx.x >> 5, qd = threadIdx.x & 31, hq = a.g_heads[grp][h];
      float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int g = 0; g < G; ++g) {
        const float4 v = sAcc[(g * nh + h) * 32 + qd];
        O.x += v.x; O.y += v.y; O.z += v.z; O.w += v.w;
      }
      const float inv = sHd[h];
      const int64_t orow = (static_cast<int64_t>(b) * a.n_q_heads + hq) * kD + 4 * qd;
      if (a.part_out != nullptr) {
        float* dst = a.part_out + (static_cast<int64_t>(b) * a.n_q_heads + hq) * kPartStride;
        if (qd == 0) *reinterpret_cast<float4*>(dst) = make_float4(sHd[SL + h], sHd[2 * SL + h], 0.f, 0.f);
        *reinterpret_cast<float4*>(dst + 4 + 4 * qd) = O;
      } else if (a.out_f32) {
        *reinterpret_cast<float4*>(static_cast<float*>(a.out) + orow) =
            make_float4(O.x * inv, O.y * inv, O.z * inv, O.w * inv);
      } else {
        __nv_bfloat162 lo = __floats2bfloat162_rn(O.x * inv, O.y * inv);
        __nv_bfloat162 hi = __floats2bfloat162_rn(O.z * inv, O.w * inv);
        uint2 pk;
        pk.x = *reinterpret_cast<uint32_t*>(&lo);
        pk.y = *reinterpret_cast<uint32_t*>(&hi);
        *reinterpret_cast<uint2*>(static_cast<uint16_t*>(a.out) + orow) = pk;
      }
    }
  }
  if (threadIdx.x == 0) a.counters[static_cast<int64_t>(b) * a.n_q_heads + a.g_heads[grp][0]] = 0;
}

template <int MB, int VB, int NH, int K, int NSET>
tq_status run_decode(const DecodeArgs& a, dim3 grid, cudaStream_t st) {
  constexpr int smem = LayPick<MB, VB, K, NSET>::type::total;
  auto kern = k_decode<MB, VB, NH, K, NSET>;
  static bool configured = false;
  if (!configured) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
        cudaSuccess)
      return TQ_ECUDA;
    configured = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(Cfg<NSET>::threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, a) != cudaSuccess) return TQ_ECUDA;
  return cudaGetLastError() == cudaSuccess ? TQ_OK : TQ_ECUDA;
}

template <int MB, int VB, int K>
tq_status run_decode_nh(const DecodeArgs& a, dim3 grid, int max_heads, cudaStream_t st) {
  if (max_heads <= 2) return run_decode<MB, VB, 2, K, 1>(a, grid, st);
  if (max_heads == 3) return run_decode<MB, VB, 3, K, 1>(a, grid, st);
  return run_decode<MB, VB, 4, K, 1>(a, grid, st);
}

// LSE merge of context-split partial records (m, l, o) of n_parts slices: per row (sequence,
// query head) M = max m_r, out = sum 2^(m_r - M) o_r / sum 2^(m_r - M) l_r (zeros when every
// slice is empty). One warp per row, lane l owns channels 4l .. 4l + 3.
__global__ void __launch_bounds__(128) k_merge_partials(const float* __restrict__ parts, int n_parts,
                                                        int64_t rows, void* out, int out_f32) {
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  float M = -INFINITY;
  for (int r = 0; r < n_parts; ++r) M = fmaxf(M, __ldg(parts + (r * rows + row) * kPartStride));
  float L = 0.f;
  float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
  if (M != -INFINITY) {
    for (int r = 0; r < n_parts; ++r) {
      const float* rec = parts + (r * rows + row) * kPartStride;
      const float mr = __ldg(rec);
      if (mr == -INFINITY) continue;
      const float f = exp2f(mr - M);
      L = fmaf(f, __ldg(rec + 1), L);
      const float4 v = __ldg(reinterpret_cast<const float4*>(rec + 4) + lane);
      O.x = fmaf(f, v.x, O.x); O.y = fmaf(f, v.y, O.y);
      O.z = fmaf(f, v.z, O.z); O.w = fmaf(f, v.w, O.w);
    }
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  const int64_t orow = row * kD + 4 * lane;
  if (out_f32) {
    *reinterpret_cast<float4*>(static_cast<float*>(out) + orow) =
        make_float4(O.x * inv, O.y * inv, O.z * inv, O.w * inv);
  } else {
    __nv_bfloat162 lo = __floats2bfloat162_rn(O.x * inv, O.y * inv);
    __nv_bfloat162 hi = __floats2bfloat162_rn(O.z * inv, O.w * inv);
    uint2 pk;
    pk.x = *reinterpret_cast<uint32_t*>(&lo);
    pk.y = *reinterpret_cast<uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(static_cast<uint16_t*>(out) + orow) = pk;
  }
}

// Two table sets (up to 8 heads per CTA, 12 warps) where the layout fits; grouped keys and
// configurations whose two-set tables exceed the shared memory keep one set.
template <int MB, int VB, int K>
constexpr bool two_sets_fit() {
  if constexpr (K == kGrp) return false;
  else return LayPick<MB, VB, K, 2>::type::fits;
}

template <int MB, int VB, int K>
tq_status run_decode_sets(const DecodeArgs& a, dim3 grid, int max_heads, bool two,
                          cudaStream_t st) {
  if constexpr (two_sets_fit<MB, VB, K>()) {
    if (two) {
      if (max_heads <= 6) return run_decode<MB, VB, 6, K, 2>(a, grid, st);
      return run_decode<MB, VB, 8, K, 2>(a, grid, st);
    }
  }
  return run_decode_nh<MB, VB, K>(a, grid, max_heads, st);
}

bool two_sets_ok(int kind, int mb, int vb) {
  switch (kind * 64 + mb * 8 + vb) {
    case kProd * 64 + 1 * 8 + 0: return two_sets_fit<1, 0, kProd>();
    case kProd * 64 + 1 * 8 + 2: return two_sets_fit<1, 2, kProd>();
    case kProd * 64 + 1 * 8 + 4: return two_sets_fit<1, 4, kProd>();
    case kProd * 64 + 2 * 8 + 0: return two_sets_fit<2, 0, kProd>();
    case kProd * 64 + 2 * 8 + 2: return two_sets_fit<2, 2, kProd>();
    case kProd * 64 + 2 * 8 + 4: return two_sets_fit<2, 4, kProd>();
    case kProd * 64 + 3 * 8 + 0: return two_sets_fit<3, 0, kProd>();
    case kProd * 64 + 3 * 8 + 2: return two_sets_fit<3, 2, kProd>();
    case kProd * 64 + 3 * 8 + 4: return two_sets_fit<3, 4, kProd>();
    case kMse * 64 + 1 * 8 + 0: return two_sets_fit<1, 0, kMse>();
    case kMse * 64 + 1 * 8 + 2: return two_sets_fit<1, 2, kMse>();
    case kMse * 64 + 1 * 8 + 4: return two_sets_fit<1, 4, kMse>();
    case kMse * 64 + 2 * 8 + 0: return two_sets_fit<2, 0, kMse>();
    case kMse * 64 + 2 * 8 + 2: return two_sets_fit<2, 2, kMse>();
    case kMse * 64 + 2 * 8 + 4: return two_sets_fit<2, 4, kMse>();
    case kMse * 64 + 3 * 8 + 0: return two_sets_fit<3, 0, kMse>();
    case kMse * 64 + 3 * 8 + 2: return two_sets_fit<3, 2, kMse>();
    case kMse * 64 + 3 * 8 + 4: return two_sets_fit<3, 4, kMse>();
    case kMse * 64 + 4 * 8 + 0: return two_sets_fit<4, 0, kMse>();
    case kMse * 64 + 4 * 8 + 2: return two_sets_fit<4, 2, kMse>();
    case kMse * 64 + 4 * 8 + 4: return two_sets_fit<4, 4, kMse>();
    case kGrp * 64 + 1 * 8 + 0: return two_sets_fit<1, 0, kGrp>();
    case kGrp * 64 + 1 * 8 + 2: return two_sets_fit<1, 2, kGrp>();
    case kGrp * 64 + 1 * 8 + 4: return two_sets_fit<1, 4, kGrp>();
    case kGrp * 64 + 2 * 8 + 0: return two_sets_fit<2, 0, kGrp>();
    case kGrp * 64 + 2 * 8 + 2: return two_sets_fit<2, 2, kGrp>();
    case kGrp * 64 + 2 * 8 + 4: return two_sets_fit<2, 4, kGrp>();
    case kGrp * 64 + 3 * 8 + 0: return two_sets_fit<3, 0, kGrp>();
    case kGrp * 64 + 3 * 8 + 2: return two_sets_fit<3, 2, kGrp>();
    case kGrp * 64 + 3 * 8 + 4: return two_sets_fit<3, 4, kGrp>();
    default: return false;
  }
}

int max_splits_for(int capacity) {
  const int s = (capacity + 255) / 256;
  return s < 1 ? 1 : (s > 256 ? 256 : s);
}

}  // namespace

tq_status launch_merge_partials(const float* parts, int n_parts, int64_t rows, void* out,
                                int out_dtype, cudaStream_t st) {
  if (rows == 0) return TQ_OK;
  const int64_t blocks = (rows + 3) / 4;
  k_merge_partials<<<static_cast<unsigned>(blocks), 128, 0, st>>>(parts, n_parts, rows, out,
                                                                 out_dtype == TQ_F32);
  return cudaGetLastError() == cudaSuccess ? TQ_OK : TQ_ECUDA;
}

size_t decode_workspace_bytes(int batch, int n_q_heads, int capacity) {
  const size_t parts = static_cast<size_t>(batch) * n_q_heads * max_splits_for(capacity) *
                       kPartStride * sizeof(float);
  const size_t ctrs = static_cast<size_t>(batch) * n_q_heads * sizeof(int);
  return ((parts + 255) / 256) * 256 + ((ctrs + 255) / 256) * 256;
}

tq_status launch_decode(const tq_quantizer* q, const tq_kv_cache* c, const void* qv, int q_dtype,
                        int n_q_heads, const int32_t* head_map, float sm_scale, void* out,
                        int out_dtype, float* scores, int64_t scores_ld, float* part_out,
                        void* workspace, size_t workspace_bytes, cudaStream_t st) {
  DecodeArgs a{};
  a.part_out = part_out;
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

  // key kind and widths (MB: index bits, prod: bits - 1; grouped: the base bits)
  const int kind = q->mode == TQ_MODE_PROD ? kProd : (q->mode == TQ_MODE_GROUPED ? kGrp : kMse);
  const int mb = kind == kProd ? q->bits - 1 : q->bits;
  const int vb = c->value_bits;

  int max_len = 0;
  for (int b = 0; b < c->batch; ++b) max_len = c->len_host[b] > max_len ? c->len_host[b] : max_len;
  int dev = 0;
  cudaGetDevice(&dev);
  const int sms = std::max(1, sm_count(dev) - 4);

  // The query heads of each KV head; a CTA serves up to 8 of them (two table sets) where some
  // KV head has more than 4, the two-set layout fits, and the decode is large enough to
  // amortise the two-set CTA's longer fixed path (its prologue builds twice the tables and
  // its chunks carry twice the heads): at least 4 chunk rounds of (token, KV head) units per
  // SM. Measured: 1.05 M units (batch 8 x 4 KV heads x 32768, or 1 x 8 x 131072) run 11-16 %
  // faster with two sets; 65536 units (1 x 2 x 32768) run 16 % slower. tq_set_decode_policy
  // can force either shape.
  int per_kv_max = 0;
  for (int kv = 0; kv < c->n_kv_heads; ++kv) {
    int n = 0;
    for (int h = 0; h < n_q_heads; ++h)
      if ((head_map ? head_map[h] : h / (n_q_heads / c->n_kv_heads)) == kv) ++n;
    per_kv_max = n > per_kv_max ? n : per_kv_max;
  }
  const long long units = static_cast<long long>(c->batch) * c->n_kv_heads * max_len;
  const int policy = g_decode_policy.load(std::memory_order_relaxed);
  const bool two = per_kv_max > kMaxHeads && two_sets_ok(kind, mb, vb) &&
                   policy != TQ_DECODE_ONE_SET &&
                   (policy == TQ_DECODE_TWO_SETS || units >= 4ll * Cfg<2>::chunk_stride * sms);
  const int cap = two ? kMaxSlots : kMaxHeads;
  // head groups: the query heads of each KV head, in balanced groups of at most `cap`
  int n_groups = 0, max_heads = 0;
  for (int kv = 0; kv < c->n_kv_heads; ++kv) {
    int heads[1024];
    int n = 0;
    for (int h = 0; h < n_q_heads; ++h)
      if ((head_map ? head_map[h] : h / (n_q_heads / c->n_kv_heads)) == kv) heads[n++] = h;
    if (n == 0) continue;
    const int ng = (n + cap - 1) / cap;
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

  if (max_len == 0 && out == nullptr && part_out == nullptr) return TQ_OK;

  // split count: one CTA per SM; minimise waves x (tokens per split + per-CTA set-up) + the
  // final combine (its loads grow with the number of splits). A few SMs are left out of the
  // first wave so that an append kernel still resident on them does not hold back a CTA of
  // this grid when it starts early (programmatic dependent launch).
  const int pairs = c->batch * n_groups;
  const int cap_splits = max_splits_for(c->capacity);
  int best = 1;
  double best_cost = 1e300;
  const int max_try = std::max(1, std::min(cap_splits, (max_len + 255) / 256));
  for (int s = 1; s <= max_try; ++s) {
    const int tps = ((max_len + s - 1) / s + 31) & ~31;
    const int used = (max_len + tps - 1) / tps;
    if (used != s) continue;
    const double waves = std::ceil(static_cast<double>(pairs) * s / sms);
    const double cost = waves * (tps + (two ? Cfg<2>::chunk_stride : Cfg<1>::chunk_stride)) +
                        (s > 1 ? 8.0 * s : 0.0);
    if (cost < best_cost - 1e-9) { best_cost = cost; best = s; }
  }
  a.n_splits = best;
  a.max_len = max_len;
  a.tokens_per_split = std::max(32, ((max_len + best - 1) / best + 31) & ~31);
  if (decode_workspace_bytes(c->batch, n_q_heads, c->capacity) > workspace_bytes) return TQ_EINVAL;
  const size_t parts = static_cast<size_t>(c->batch) * n_q_heads * cap_splits * kPartStride * sizeof(float);
  a.part = static_cast<float*>(workspace);
  a.counters = reinterpret_cast<int*>(static_cast<uint8_t*>(workspace) + ((parts + 255) / 256) * 256);

  const dim3 grid(a.n_splits, n_groups, c->batch);
  switch (kind * 64 + mb * 8 + vb) {
    case kProd * 64 + 1 * 8 + 0: return run_decode_sets<1, 0, kProd>(a, grid, max_heads, two, st);
    case kProd * 64 + 1 * 8 + 2: return run_decode_sets<1, 2, kProd>(a, grid, max_heads, two, st);
    case kProd * 64 + 1 * 8 + 4: return run_decode_sets<1, 4, kProd>(a, grid, max_heads, two, st);
    case kProd * 64 + 2 * 8 + 0: return run_decode_sets<2, 0, kProd>(a, grid, max_heads, two, st);
    case kProd * 64 + 2 * 8 + 2: return run_decode_sets<2, 2, kProd>(a, grid, max_heads, two, st);
    case kProd * 64 + 2 * 8 + 4: return run_decode_sets<2, 4, kProd>(a, grid, max_heads, two, st);
    case kProd * 64 + 3 * 8 + 0: return run_decode_sets<3, 0, kProd>(a, grid, max_heads, two, st);
    case kProd * 64 + 3 * 8 + 2: return run_decode_sets<3, 2, kProd>(a, grid, max_heads, two, st);
    case kProd * 64 + 3 * 8 + 4: return run_decode_sets<3, 4, kProd>(a, grid, max_heads, two, st);
    case kMse * 64 + 1 * 8 + 0: return run_decode_sets<1, 0, kMse>(a, grid, max_heads, two, st);
    case kMse * 64 + 1 * 8 + 2: return run_decode_sets<1, 2, kMse>(a, grid, max_heads, two, st);
    case kMse * 64 + 1 * 8 + 4: return run_decode_sets<1, 4, kMse>(a, grid, max_heads, two, st);
    case kMse * 64 + 2 * 8 + 0: return run_decode_sets<2, 0, kMse>(a, grid, max_heads, two, st);
    case kMse * 64 + 2 * 8 + 2: return run_decode_sets<2, 2, kMse>(a, grid, max_heads, two, st);
    case kMse * 64 + 2 * 8 + 4: return run_decode_sets<2, 4, kMse>(a, grid, max_heads, two, st);
    case kMse * 64 + 3 * 8 + 0: return run_decode_sets<3, 0, kMse>(a, grid, max_heads, two, st);
    case kMse * 64 + 3 * 8 + 2: return run_decode_sets<3, 2, kMse>(a, grid, max_heads, two, st);
    case kMse * 64 + 3 * 8 + 4: return run_decode_sets<3, 4, kMse>(a, grid, max_heads, two, st);
    case kMse * 64 + 4 * 8 + 0: return run_decode_sets<4, 0, kMse>(a, grid, max_heads, two, st);
    case kMse * 64 + 4 * 8 + 2: return run_decode_sets<4, 2, kMse>(a, grid, max_heads, two, st);
    case kMse * 64 + 4 * 8 + 4: return run_decode_sets<4, 4, kMse>(a, grid, max_heads, two, st);
    case kGrp * 64 + 1 * 8 + 0: return run_decode_sets<1, 0, kGrp>(a, grid, max_heads, two, st);
    case kGrp * 64 + 1 * 8 + 2: return run_decode_sets<1, 2, kGrp>(a, grid, max_heads, two, st);
    case kGrp * 64 + 1 * 8 + 4: return run_decode_sets<1, 4, kGrp>(a, grid, max_heads, two, st);
    case kGrp * 64 + 2 * 8 + 0: return run_decode_sets<2, 0, kGrp>(a, grid, max_heads, two, st);
    case kGrp * 64 + 2 * 8 + 2: return run_decode_sets<2, 2, kGrp>(a, grid, max_heads, two, st);
    case kGrp * 64 + 2 * 8 + 4: return run_decode_sets<2, 4, kGrp>(a, grid, max_heads, two, st);
    case kGrp * 64 + 3 * 8 + 0: return run_decode_sets<3, 0, kGrp>(a, grid, max_heads, two, st);
    case kGrp * 64 + 3 * 8 + 2: return run_decode_sets<3, 2, kGrp>(a, grid, max_heads, two, st);
    case kGrp * 64 + 3 * 8 + 4: return run_decode_sets<3, 4, kGrp>(a, grid, max_heads, two, st);
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
                       scores_ld, nullptr, base, need, st);
}

tq_status set_decode_policy(int policy, int* previous) {
  if (policy != TQ_DECODE_AUTO && policy != TQ_DECODE_ONE_SET && policy != TQ_DECODE_TWO_SETS)
    return TQ_EINVAL;
  const int old = g_decode_policy.exchange(policy);
  if (previous) *previous = old;
  return TQ_OK;
}

}  // namespace tq
