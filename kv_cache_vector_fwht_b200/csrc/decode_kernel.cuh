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
// 1-bit index byte 8, a byte of two 4-bit or two 3-bit (nibble) indices 2, a QJL sign byte
// 8. The Lloyd-Max codebook is symmetric (C[L-1-k] = -C[k]) and the sign sums are odd, so a
// byte and its mirror (every code k -> L-1-k, every sign flipped) differ only in sign: a
// table keeps the canonical half (bytes 0..127; for 3-bit nibble bytes 0..0x37, the high
// code below 4) and a lookup returns (entry, +-1). An entry holds the partial sums of 4
// query heads (16 bytes, one table set); a block holds one or two sets. Entry e of position
// p sits at (e * P + p) * 16 bytes of its set. At step i of an 8-position block, lane l reads
// position 8 b + ((l + i) mod 8), so the eight lanes of one 16-byte shared-memory phase fall
// in eight different bank groups. Tables are pre-multiplied by sm_scale * log2(e): the
// online softmax runs in base 2.
//
// Grid: (context split, head group, sequence); a block takes one KV head, up to 4 (one set)
// or 8 (two sets) of its query heads and a contiguous token range. Warp w walks its own
// 32-token chunks (chunk w, w + W, ... of the range), so no block-wide barrier sits in the
// loop. Per chunk:
//   scores   lane = token: the token's key bytes and value parameters (prefetched one chunk
//            ahead in registers), one lookup per byte and set, the two norms;
//   softmax  per head a warp-uniform reference maximum m that is raised only when some
//            score exceeds it by more than kTau (a vote, not a reduction, in the common
//            case); p = 2^(s - m) <= 2^kTau; the lane's sum l and its largest score;
//   P.V      the chunk's value codes arrive in the warp's shared slot by cp.async; the two
//            half-warps take alternate tokens, lane j of a half owns channels 8j .. 8j + 7,
//            dequantizes them once (v = (1 + code/16) * 16 s16 + (mn16 - 16 s16), exact
//            field insertion and one packed FMA per channel pair) and accumulates every head
//            in packed fp32x2 FMAs; the token's p of 4 heads is one shared 16-byte
//            broadcast and each head's (p, p) operand pair is formed in registers.
// Each block merges its warps and writes a partial (m, l, o) with m the largest logit; the
// last block of a (sequence, head group) to finish merges all partials (an atomic counter,
// no waiting), or writes the merged partial itself for a context-parallel decode.
#pragma once

#include <cfloat>
#include <cmath>

#include "tq_device.cuh"
#include "tq_internal.h"

namespace tq {
namespace dec {

constexpr int kSetHeads = 4;       // query heads of one table set (one 16-byte entry)
constexpr int kMaxSlots = 8;       // query heads of a block: at most two table sets
constexpr int kMaxGroups = 256;    // head groups of one launch
constexpr int kMaxQHeads = 512;
constexpr int kPartStride = 132;   // floats per (head, split) partial: m, l, pad, o[128]
constexpr int kVpStride = 34;      // value parameters of a warp's chunk: [group][34 tokens]
constexpr int kQStride = 272;      // bytes per staged fp16 query row (256 + 16: bank spread)
constexpr float kTau = 8.f;        // lazy rescale threshold of the online softmax (base 2)

enum KeyKind { kMse = 0, kProd = 1, kGrp = 2 };

// A head group: KV head (bits 0-15), index of its first query head in DecodeArgs::heads
// (bits 16-25), number of query heads (bits 26-29).
__host__ __device__ constexpr uint32_t group_word(int kv, int first, int n) {
  return static_cast<uint32_t>(kv) | (static_cast<uint32_t>(first) << 16) |
         (static_cast<uint32_t>(n) << 26);
}

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
  int* err;         // device error word (bounded waits that ran out); see tq_sync_status
  const DevTables* tab;
  int64_t scores_ld;
  int n_kv_heads, capacity, n_q_heads;
  int q_f32, out_f32;
  int n_splits, tokens_per_split;
  int max_len;  // host copy of the longest sequence (an upper bound of every len[b])
  float scale_log2, inv_scale_log2;
  uint32_t group[kMaxGroups];
  int16_t heads[kMaxQHeads];  // query heads in group order
};

// Block shape for NSET table sets: 16 warps with one set (up to 4 heads, 4 accumulator pairs
// per head and lane); 8 warps with two sets (up to 8 heads: 64 accumulator registers a lane,
// and two sets of tables in the shared memory).
template <int NSET>
struct Shape {
  static constexpr int slots = kSetHeads * NSET;
  static constexpr int warps = NSET == 1 ? 16 : 8;
  static constexpr int threads = 32 * warps;
  static constexpr int chunk_stride = 32 * warps;  // tokens between a warp's chunks
};

__host__ __device__ constexpr int round_up(int x, int m) { return (x + m - 1) / m * m; }

// Shared-memory plan. MB: index bits (mse, prod) or the grouped base bits b. A token's key
// bytes form two lookup segments: I (index bytes; grouped: the outlier group) and S (prod:
// the QJL sign bytes; grouped: the normal group, padded with zero bytes to whole 8-byte
// blocks). Each segment accumulates its own sum; the two norms scale them.
// A warp's per-head record after the main loop (floats): m at 0, the lanes' sums from
// kWRecL, their largest logits from kWRecX, the two half-warps' outputs from kWRecO.
constexpr int kWRecL = 4, kWRecX = kWRecL + 32, kWRecO = kWRecX + 32, kWRec = kWRecO + 2 * kD;

template <int MB, int VB, int K, int NSET, int NH>
struct Lay {
  static constexpr int SL = Shape<NSET>::slots, NW = Shape<NSET>::warps;
  static constexpr bool GRP = K == kGrp;
  static constexpr int MI = GRP ? MB + 1 : MB;                      // segment I code bits
  static constexpr int MS = GRP ? MB : 1;                           // segment S code bits
  static constexpr int IBI = (GRP ? 32 : kD) * storage_width_c(MI) / 8;
  static constexpr int IBS = GRP ? 96 * storage_width_c(MS) / 8 : 0;
  static constexpr int IB = IBI + IBS;                              // index-plane bytes
  static constexpr int PI = IBI;                                    // segment I positions
  static constexpr int EI = MI == 3 ? 56 : 128;                     // canonical entries
  static constexpr int PS = K == kProd ? 16 : (GRP ? round_up(IBS, 8) : 0);
  static constexpr int ES = MS == 3 ? 56 : 128;
  static constexpr int KW = (IBI + (GRP ? PS : 0)) / 4;             // key words held a token
  static constexpr int NB = K == kMse ? 2 : 4;                      // norm bytes per token
  static constexpr int VQB = VB ? kD * VB / 8 : 0;                  // value code bytes
  static constexpr int SETI = EI * PI * 16;                         // bytes of one index set
  static constexpr int SETS = ES * PS * 16;                         // bytes of one S set
  static constexpr int lutI = 0;
  static constexpr int lutS = lutI + NSET * SETI;
  static constexpr int tables = lutS + NSET * SETS;
  // per-warp slot: softmax weights p of 4 heads a float4 [NH4][32], value parameters [4][kVpStride],
  // value codes [32][VQB]
  static constexpr int NH4 = (NH + 3) / 4;
  static constexpr int oPP = 0;
  static constexpr int oVP = oPP + NH4 * 32 * 16;
  static constexpr int wv = round_up(tables, 128);
  static constexpr int budget = 227 * 1024 - 512;                  // leave room for static smem
  // value parameters as float4 (16 s16-scaled pairs and offsets) where the slots fit, else
  // as float2 (s16, mn16) with the pairs formed in the P.V loop
  static constexpr bool VP4 =
      wv + NW * round_up(oVP + 4 * kVpStride * 16 + 32 * VQB, 128) <= budget;
  static constexpr int oVQ = oVP + 4 * kVpStride * (VP4 ? 16 : 8);
  static constexpr int WB = round_up(oVQ + 32 * VQB, 128);
  static constexpr int warps_end = wv + NW * WB;
  // prologue scratch over the warp slots: q_rot and Sq [128][SL] f32, fp16 hi / lo query rows
  static constexpr int qrT = wv;
  static constexpr int sqT = qrT + kD * SL * 4;
  static constexpr int qhi = sqT + kD * SL * 4;
  static constexpr int qlo = qhi + 8 * kQStride;
  static constexpr int qinv = qlo + 8 * kQStride;
  static constexpr int pro_end = qinv + 32;
  // after the main loop, from byte 0: the warps' records [NW][SL][kWRec] f32, or the
  // last block's slice maxima and sums and slice partial outputs
  static constexpr int merge = NW * SL * kWRec * 4;
  static constexpr int last = 16 * 8 * SL + NW * SL * 32 * 16;
  static constexpr int total0 = warps_end > pro_end ? warps_end : pro_end;
  static constexpr int total1 = total0 > merge ? total0 : merge;
  static constexpr int total = total1 > last ? total1 : last;
  static_assert(IBI % 8 == 0 && PS % 8 == 0, "whole 8-byte lookup blocks");
  static constexpr bool fits = total <= budget;
};

// Programmatic dependent launch: wait until the grids this one depends on have completed and
// their memory is visible (a no-op when the kernel was launched without the attribute).
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// (+1.0, +1.0) or (-1.0, -1.0) from an all-ones / all-zeros mask
__device__ __forceinline__ uint64_t sign_pair(int mask) {
  const float s = __uint_as_float(0x3f800000u | (static_cast<uint32_t>(mask) & 0x80000000u));
  return pk2(s, s);
}

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

// Lookups of one 8-byte block of bytes whose mirror is the bitwise complement (index bytes
// of 1-, 2- or 4-bit codes, or sign bytes): byte i of the rotated block is position
// 8 blk + ((l + i) mod 8).
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

// Lookups of one 8-byte block of bytes holding two 3-bit codes in their nibbles (bits 3 and
// 7 clear): the mirror flips both codes (k -> 7 - k, the byte XOR 0x77) and is taken when
// bit 6 is set (high code >= 4); the canonical byte (0..0x37) is the entry index.
template <int ROWB, int NS, int SETB>
__device__ __forceinline__ void block_lookups3(uint64_t (&acc)[NS][2], uint32_t R0, uint32_t R1,
                                               const uint8_t* tab, int blk,
                                               const uint32_t (&rot16)[8]) {
  const uint32_t S0 = R0 << 1, S1 = R1 << 1;  // bit 7 of every byte is clear: no carries
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t R = i < 4 ? R0 : R1;
    const uint32_t R2 = i < 4 ? S0 : S1;
    // byte i zero-extended, and the mirror flag (bit 6, moved to bit 7 in R << 1) replicated
    // over a word: one byte permute each
    uint32_t v, ms;
    asm("prmt.b32 %0, %1, 0, %2;" : "=r"(v) : "r"(R), "r"(static_cast<uint32_t>((i & 3) | 0x4440)));
    asm("prmt.b32 %0, %1, 0, %2;" : "=r"(ms) : "r"(R2), "r"(static_cast<uint32_t>((8 | (i & 3)) * 0x1111)));
    const int msk = static_cast<int>(ms);
    const uint32_t e = v ^ (ms & 0x77u);
    lut_acc<NS, SETB>(acc, tab + 128 * blk + e * ROWB + rot16[i], sign_pair(msk));
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
    // 3-bit nibble bytes: bits 3 and 7 cleared, which keeps every entry index in the table
    // whatever the bytes hold
    constexpr uint32_t wm = MBITS == 3 ? 0x77777777u : 0xffffffffu;
    rot_block(w[2 * blk] & wm, w[2 * blk + 1] & wm, swap, sh, R0, R1);
    if constexpr (MBITS == 3) block_lookups3<NPOS * 16, NS, SETB>(acc, R0, R1, tab, blk, rot16);
    else block_lookups<NPOS * 16, NS, SETB>(acc, R0, R1, tab, blk, rot16);
  }
}

// Float index of (coordinate j, head slot s) in a [128][SL] query array whose 16-byte units
// (4 head slots of one coordinate) are XOR-permuted by (j / XC) & 7 within aligned groups of
// 8 units: the table builders' lanes take consecutive byte positions p and read coordinate
// XC p + f at the same f, which lands them in 8 different bank groups per 128-byte phase.
template <int XC, int SL>
__device__ __forceinline__ int xidx(int j, int s) {
  const int u = j * (SL / 4) + (s >> 2);
  return 4 * (u ^ ((j / XC) & 7)) + (s & 3);
}

// Build the lookup table of one segment for table set st: NPOS positions of bytes whose
// coordinates c0 + CPB p + f (f < CPB coordinates per byte) carry CB-bit codes (CB = 0: QJL
// sign bits, value +-cs); entry e = sum_f x[coordinate][head] * cen[code_f(e)] * cs for the
// canonical bytes (top bit clear; 3-bit nibble bytes: high code below 4). x is a [128][SL]
// f32 array (q_rot or Sq; laid out by xidx<XC, SL>), 4 heads from column 4 st. An item (position, high nibble) loads
// its coordinates once, sums the high nibble's coordinates once and writes the entries of
// every low nibble, whose codes are compile-time constants (centroids from registers).
// Positions p >= nvalid are padding of the grouped normal segment and stay zero.
template <int CB, int NPOS, int SL, int XC>
__device__ __forceinline__ void build_table(uint8_t* lut, const float* x, int c0, int st,
                                            const float* cen, float cs, int nvalid, int tid,
                                            int nthreads) {
  constexpr int W = CB == 0 ? 1 : storage_width_c(CB);
  constexpr int CPB = 8 / W;              // coordinates per byte
  constexpr int HALF = CPB / 2;           // coordinates per nibble
  constexpr int NLO = CB == 3 ? 8 : 16;   // low-nibble values of a canonical byte
  constexpr int NHI = CB == 3 ? 4 : 8;    // high-nibble values of a canonical byte
  constexpr int NC = CB == 0 ? 2 : 1 << CB;
  constexpr int CM = NC - 1;
  float cv[NC];
#pragma unroll
  for (int k = 0; k < NC; ++k) cv[k] = CB == 0 ? (k ? cs : -cs) : cen[k] * cs;
  for (int it = tid; it < NPOS * NHI; it += nthreads) {
    const int p = it % NPOS, hi = it / NPOS;
    const bool ok = p < nvalid;
    float4 xs[CPB];
#pragma unroll
    for (int f = 0; f < CPB; ++f)
      xs[f] = ok ? *reinterpret_cast<const float4*>(x + xidx<XC, SL>(c0 + CPB * p + f, 4 * st))
                 : make_float4(0.f, 0.f, 0.f, 0.f);
    float4 ph = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int f = 0; f < HALF; ++f) {
      const int code = (hi >> (W * f)) & CM;
      const float c = CB == 0 ? (code ? cs : -cs) : cen[code] * cs;
      ph.x = fmaf(xs[HALF + f].x, c, ph.x);
      ph.y = fmaf(xs[HALF + f].y, c, ph.y);
      ph.z = fmaf(xs[HALF + f].z, c, ph.z);
      ph.w = fmaf(xs[HALF + f].w, c, ph.w);
    }
#pragma unroll
    for (int lo = 0; lo < NLO; ++lo) {
      float4 r = ph;
#pragma unroll
      for (int f = 0; f < HALF; ++f) {
        const float c = cv[(lo >> (W * f)) & CM];
        r.x = fmaf(xs[f].x, c, r.x);
        r.y = fmaf(xs[f].y, c, r.y);
        r.z = fmaf(xs[f].z, c, r.z);
        r.w = fmaf(xs[f].w, c, r.w);
      }
      const uint32_t e = static_cast<uint32_t>(lo | (hi << 4));
      *reinterpret_cast<float4*>(lut + (e * NPOS + p) * 16) = r;
    }
  }
}

// K = kMse: s = n16 <Pi q, c[idx]>; kProd: + r16 sqrt(pi/2)/d <S q, 2 sigma - 1>;
// kGrp: s = n_o <Pi_o q_o, c_o[idx_o]> + n_n <Pi_n q_n, c_n[idx_n]> over the two channel
// groups (Pi_g: 32-point Hadamard blocks after the group's signs).
// The query prologue of a block (it reads only the query and the quantizer's tables): q_rot =
// H (s . q) per head slot (grouped: gathered in channel order, 32-point blocks), Sq = S_rot
// q_rot / sqrt(d) on tensor cores (mma.sync, fp16 hi + lo halves of q_rot, fp32 accumulation),
// then the byte lookup tables of every set. Every thread of the block takes part; the block
// has at least 8 warps. Ends with the tables complete (a block-wide barrier).
template <class Lo, int K, int NSET, int NT>
__device__ __forceinline__ void decode_prologue(const DecodeArgs& a, uint8_t* smem, float* sCen,
                                                const int16_t* gheads, int nh, int b) {
  constexpr int SL = Lo::SL, PI = Lo::PI;
  constexpr bool PROD = K == kProd, GRP = K == kGrp;
  // coordinates per index byte: the swizzle key of q_rot (the sign tables read Sq by 8)
  constexpr int XCI = 8 / storage_width_c(Lo::MI);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint8_t* lutI = smem + Lo::lutI;
  uint8_t* lutS = smem + Lo::lutS;
  float* qrT = reinterpret_cast<float*>(smem + Lo::qrT);
  float* sqT = reinterpret_cast<float*>(smem + Lo::sqT);
  uint8_t* qhi = smem + Lo::qhi;
  uint8_t* qlo = smem + Lo::qlo;
  float* qinv = reinterpret_cast<float*>(smem + Lo::qinv);
  const DevTables* __restrict__ tab = a.tab;
  // S_rot rows [16 warp, 16 warp + 16) as mma.sync A fragments (warps 0..7)
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
      const int hq = gheads[warp];
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
      if (warp < SL) qrT[xidx<XCI, SL>(j, warp)] = v[i];
      const float sv = v[i] * scl;
      const __half hi = __float2half_rn(sv);
      const __half lo = __float2half_rn(sv - __half2float(hi));
      reinterpret_cast<__half*>(qhi + warp * kQStride)[j] = hi;
      reinterpret_cast<__half*>(qlo + warp * kQStride)[j] = lo;
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
        const uint8_t* bq = (part ? qlo : qhi) + g * kQStride;
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
      sqT[xidx<8, SL>(j0, 2 * t)] = c0 * s0;
      sqT[xidx<8, SL>(j0, 2 * t + 1)] = c1 * s1;
      sqT[xidx<8, SL>(j0 + 8, 2 * t)] = c2 * s0;
      sqT[xidx<8, SL>(j0 + 8, 2 * t + 1)] = c3 * s1;
    }
  }
  if constexpr (PROD) __syncthreads();
  {
    // entry scales: 1/sqrt(d) of Pi times 1/sqrt(d) of the N(0,1)-scale centroids (grouped:
    // 1/sqrt(32) of a Hadamard block times 1/sqrt(d_g)); prod signs: sqrt(pi/2)/d
    const float cI = a.scale_log2 * (GRP ? 1.f / 32.f : 1.f / 128.f);
    const float cS = GRP ? a.scale_log2 * 0.018042195912175807f
                         : a.scale_log2 * 1.2533141373155002512f / 128.f;
#pragma unroll
    for (int st = 0; st < NSET; ++st) {
      build_table<Lo::MI, PI, SL, XCI>(lutI + st * Lo::SETI, qrT, 0, st, sCen, cI, PI, threadIdx.x, NT);
      if constexpr (PROD)
        build_table<0, 16, SL, 8>(lutS + st * Lo::SETS, sqT, 0, st, sCen, cS, 16, threadIdx.x, NT);
      if constexpr (GRP)
        build_table<Lo::MS, Lo::PS, SL, XCI>(lutS + st * Lo::SETS, qrT, 32, st, sCen + 16, cS,
                                        Lo::IBS, threadIdx.x, NT);
    }
  }
  __syncthreads();
}

// The block's partial from its warps' NREC records [NREC][SL][kWRec] at smem (m: the warp's
// reference maximum; per lane: its sum relative to m and its largest logit; the outputs of
// the two half-warps, 128 channels each):
// relative to the block's largest logit M, written as the output (one split), as a
// context-parallel record, or as a split partial; the last block of a (sequence, head group)
// to finish then merges every split. Every thread of the block calls this.
// Last-block merge scratch: slice (M, L) pairs at 0, slice outputs from kMergeAccOff (at most
// 16 slices).
template <int SL>
__host__ __device__ constexpr int kMergeAccOff() { return 16 * 8 * SL; }

template <int NH, int SL, int NT, int NREC>
__device__ __forceinline__ void decode_merge(const DecodeArgs& a, uint8_t* smem, int* sLastp,
                                             const int16_t* gheads, int nh, int b, int split) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int& sLast = *sLastp;
  float* sM = reinterpret_cast<float*>(smem);
  __syncthreads();
  if (warp < nh) {
    // partial of this block relative to its largest logit M, from the warps' records (lane:
    // channels 4 lane .. 4 lane + 3); an empty record (m = -inf, l = 0, o = 0) gets weight 0
    const int h = warp, hq = gheads[h];
    float mloc = -INFINITY;
#pragma unroll
    for (int w = 0; w < NREC; ++w) mloc = fmaxf(mloc, sM[(w * SL + h) * kWRec + kWRecX + lane]);
    const float M = warp_max(mloc);
    float Lp = 0.f, O[4] = {0.f, 0.f, 0.f, 0.f};
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < NREC; ++w) {
        const float* src = sM + (w * SL + h) * kWRec;
        const float f = ex2(src[0] - M);
        Lp = fmaf(f, src[kWRecL + lane], Lp);
        const float4 o0 = *reinterpret_cast<const float4*>(src + kWRecO + 4 * lane);
        const float4 o1 = *reinterpret_cast<const float4*>(src + kWRecO + kD + 4 * lane);
        O[0] = fmaf(f, o0.x + o1.x, O[0]);
        O[1] = fmaf(f, o0.y + o1.y, O[1]);
        O[2] = fmaf(f, o0.z + o1.z, O[2]);
        O[3] = fmaf(f, o0.w + o1.w, O[3]);
      }
    }
    const float Lsum = warp_sum(Lp);
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

  // ---------------- the last block of this (sequence, head group) merges all splits
  // One thread releases the block's partials (ordered before it by the barrier) and counts
  // the block; the last block's thread acquires the other blocks' partials before the
  // barrier that releases its readers.
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    int* ctr = a.counters + static_cast<int64_t>(b) * a.n_q_heads + gheads[0];
    const bool last = atomicAdd(ctr, 1) == a.n_splits - 1;
    if (last) __threadfence();
    sLast = last;
  }
  __syncthreads();
  if (!sLast) return;
  // Item (head, channel quad, split slice) loads the (maximum, sum, output quad) records of
  // its splits in batches of 16 (one round trip each) and merges them
  // relative to their largest maximum; the slices are then merged in shared memory.
  {
    const int S = a.n_splits;
    const int G = NT / (32 * nh);  // split slices
    float2* sML = reinterpret_cast<float2*>(smem);                        // [slice][head] (M, L)
    float4* sAcc = reinterpret_cast<float4*>(smem + kMergeAccOff<SL>());  // [slice][head][32]
    const float* base = a.part + static_cast<int64_t>(b) * a.n_q_heads * S * kPartStride;
    if (threadIdx.x < G * 32 * nh) {
      const int h = threadIdx.x / (32 * G), r = threadIdx.x - h * 32 * G;
      const int qd = r & 31, g = r >> 5;
      const float* src = base + static_cast<int64_t>(gheads[h]) * S * kPartStride;
      float M = -INFINITY, L = 0.f;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      constexpr int U = 16;
      for (int sp0 = g; sp0 < S; sp0 += U * G) {
        float2 ml[U];
        float4 v[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int sp = sp0 + u * G;
          if (sp < S) {
            const float* rec = src + static_cast<int64_t>(sp) * kPartStride;
            ml[u] = __ldcg(reinterpret_cast<const float2*>(rec));
            v[u] = __ldcg(reinterpret_cast<const float4*>(rec + 4 + 4 * qd));
          } else {
            ml[u] = make_float2(-INFINITY, 0.f);
            v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
          }
        }
        float mb = M;
#pragma unroll
        for (int u = 0; u < U; ++u) mb = fmaxf(mb, ml[u].x);
        if (mb == -INFINITY) continue;  // no token so far
        const float al = ex2(M - mb);   // 0 while M = -inf
        L *= al;
        acc.x *= al; acc.y *= al; acc.z *= al; acc.w *= al;
        M = mb;
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const float f = ex2(ml[u].x - M);  // 0 for an empty split (m = -inf)
          L = fmaf(f, ml[u].y, L);
          acc.x = fmaf(f, v[u].x, acc.x); acc.y = fmaf(f, v[u].y, acc.y);
          acc.z = fmaf(f, v[u].z, acc.z); acc.w = fmaf(f, v[u].w, acc.w);
        }
      }
      if (qd == 0) sML[g * SL + h] = make_float2(M, L);
      sAcc[(g * SL + h) * 32 + qd] = acc;
    }
    __syncthreads();
    if (threadIdx.x < 32 * nh) {
      const int h = threadIdx.x >> 5, qd = threadIdx.x & 31, hq = gheads[h];
      float Mt = -INFINITY;
      for (int g = 0; g < G; ++g) Mt = fmaxf(Mt, sML[g * SL + h].x);
      float Lt = 0.f;
      float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
      if (Mt != -INFINITY) {
        for (int g = 0; g < G; ++g) {
          const float2 ml = sML[g * SL + h];
          const float f = ex2(ml.x - Mt);
          const float4 v = sAcc[(g * SL + h) * 32 + qd];
          Lt = fmaf(f, ml.y, Lt);
          O.x = fmaf(f, v.x, O.x); O.y = fmaf(f, v.y, O.y);
          O.z = fmaf(f, v.z, O.z); O.w = fmaf(f, v.w, O.w);
        }
      }
      const float inv = Lt > 0.f ? 1.f / Lt : 0.f;
      const int64_t orow = (static_cast<int64_t>(b) * a.n_q_heads + hq) * kD + 4 * qd;
      if (a.part_out != nullptr) {
        float* dst = a.part_out + (static_cast<int64_t>(b) * a.n_q_heads + hq) * kPartStride;
        if (qd == 0) *reinterpret_cast<float4*>(dst) = make_float4(Mt, Lt, 0.f, 0.f);
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
  if (threadIdx.x == 0) a.counters[static_cast<int64_t>(b) * a.n_q_heads + gheads[0]] = 0;
}

template <int MB, int VB, int NH, int K, int NSET>
__global__ void __launch_bounds__(Shape<NSET>::threads, 1) k_decode(const __grid_constant__ DecodeArgs a) {
  using Lo = Lay<MB, VB, K, NSET, NH>;
  constexpr int NT = Shape<NSET>::threads, NWp = Shape<NSET>::warps;
  constexpr int CS = Shape<NSET>::chunk_stride;
  constexpr int SL = Shape<NSET>::slots;
  constexpr bool PROD = K == kProd, GRP = K == kGrp, TWO = K != kMse;
  constexpr int IB = Lo::IB, PI = Lo::PI, KW = Lo::KW, NH4 = Lo::NH4;
  static_assert(NH >= 1 && NH <= SL, "heads per block");
  static_assert(Lo::fits, "decode shared memory budget");
  constexpr bool HAS_V = VB != 0;
  extern __shared__ __align__(128) uint8_t smem[];
  const uint8_t* lutI = smem + Lo::lutI;
  const uint8_t* lutS = smem + Lo::lutS;
  __shared__ int sLast;
  __shared__ float sCen[32];

  const int split = blockIdx.x, grp = blockIdx.y, b = blockIdx.z;
  const uint32_t gw = a.group[grp];
  const int kv = static_cast<int>(gw & 0xffffu);
  const int16_t* gheads = a.heads + ((gw >> 16) & 0x3ffu);
  const int nh = static_cast<int>((gw >> 26) & 0xfu);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int t0 = split * a.tokens_per_split;
  const int64_t kvrow = (static_cast<int64_t>(b) * a.n_kv_heads + kv) * a.capacity;

  float m[NH], l[NH], mx[NH];
  uint64_t o[NH][4];
#pragma unroll
  for (int h = 0; h < NH; ++h) {
    m[h] = -INFINITY;
    l[h] = 0.f;
    mx[h] = -INFINITY;
#pragma unroll
    for (int k = 0; k < 4; ++k) o[h][k] = 0ull;
  }

  // The prologue reads only the query and the quantizer's tables, so it runs before the
  // grid-dependency wait: launched right after the library's append kernel (tq_append_decode),
  // it overlaps that kernel. The lengths and the cache are read after the wait.
  int t1 = t0;
  if (t0 < a.max_len) {
    // L2 prefetch of each warp's first chunk (its lanes spread the 128-byte lines of the five
    // planes), which lands during the prologue; every later chunk's rows are loaded one chunk
    // ahead. (Warming L2 with the block's whole token range instead kept the issuing warps
    // busy for microseconds, and its lines were read long before their use.) The rows lie
    // below the capacity; the reads proper come after the dependency wait (L2 is the point of
    // coherence for the append).
    {
      const int cf = t0 + 32 * warp;
      const int nf = min(32, min(a.max_len, t0 + a.tokens_per_split) - cf);
      if (nf > 0) {
        const uint8_t* base[5] = {a.k_idx + (kvrow + cf) * IB, a.k_sgn + (kvrow + cf) * 16,
                                  reinterpret_cast<const uint8_t*>(a.k_nrm) + (kvrow + cf) * Lo::NB,
                                  a.v_q + (kvrow + cf) * Lo::VQB,
                                  reinterpret_cast<const uint8_t*>(a.v_par) + (kvrow + cf) * 16};
        const int len[5] = {nf * IB, PROD ? nf * 16 : 0, nf * Lo::NB, nf * Lo::VQB, VB ? nf * 16 : 0};
#pragma unroll
        for (int r = 0; r < 5; ++r)
          for (int off = 128 * lane; off < len[r]; off += 32 * 128)
            asm volatile("prefetch.global.L2 [%0];" ::"l"(base[r] + off));
      }
    }

    // ---------------- prologue: rotate q, project with S_rot, build the tables
    decode_prologue<Lo, K, NSET, NT>(a, smem, sCen, gheads, nh, b);
    grid_dependency_wait();
    t1 = min(a.len[b], t0 + a.tokens_per_split);

    // ---------------- main loop over this warp's chunks
    uint8_t* wslot = smem + Lo::wv + warp * Lo::WB;
    float4* sP4 = reinterpret_cast<float4*>(wslot + Lo::oPP);     // [NH4][32] p of 4 heads
    uint8_t* sVP = wslot + Lo::oVP;                               // [4][kVpStride] params
    uint8_t* sVQ = wslot + Lo::oVQ;                               // [32][VQB]
    const uint8_t* vq_rows = a.v_q + kvrow * Lo::VQB;
    const uint16_t* vp_rows = a.v_par + kvrow * 8;
    // value dequantization of a channel pair (a, b) from one shifted code word: a's code
    // lands at mantissa bit 19 (2-bit) or 15 (4-bit), b's two or four bits above it, so
    // f_a = 1 + code_a 2^-4 (2^-8), f_b = 1 + code_b 2^-2 (2^-4) and v = f S + C with
    // S = (SA s16, SB s16), C = mn16 - S
    constexpr float SA = VB == 4 ? 256.f : 16.f, SB = VB == 4 ? 16.f : 4.f;

    // key bytes, norms and value parameters of this lane's token of chunk ts (zeros past
    // the range; grouped: the normal group's words are zero-padded to whole 8-byte blocks)
    auto load_keys = [&](int ts, uint32_t (&iw)[KW], uint32_t (&sg)[4], uint32_t& nn, uint4& vp) {
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
        if constexpr (HAS_V) vp = __ldg(reinterpret_cast<const uint4*>(vp_rows) + t);
        else vp = make_uint4(0u, 0u, 0u, 0u);
      } else {
#pragma unroll
        for (int i = 0; i < IB / 4; ++i) iw[i] = 0u;
        sg[0] = sg[1] = sg[2] = sg[3] = 0u;
        nn = 0u;
        vp = make_uint4(0u, 0u, 0u, 0u);
      }
    };
    // value codes of chunk ts into this warp's slot (cp.async, 16-byte pieces)
    auto load_codes = [&](int ts) {
      if constexpr (HAS_V) {
        const int n = min(32, t1 - ts);  // tokens of the chunk (>= 1)
        const int cq = n * Lo::VQB / 16;
        for (int c = lane; c < cq; c += 32)
          cp_async16(sVQ + 16 * c, vq_rows + static_cast<int64_t>(ts) * Lo::VQB + 16 * c, true);
      }
      cp_async_commit();
    };

    const int c0 = t0 + 32 * warp;
    uint32_t kw[KW], sw4[4], nw;
    uint4 vpar;
    if (c0 < t1) {
      load_keys(c0, kw, sw4, nw, vpar);
      load_codes(c0);
    }
    const uint32_t r8 = static_cast<uint32_t>(lane & 7);
    const bool swap = r8 >= 4;
    const uint32_t sh = 8 * (r8 & 3);
    uint32_t rot16[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) rot16[i] = ((r8 + i) & 7) * 16;
    const int hw = lane >> 4, j16 = lane & 15, vg = j16 >> 2;

    for (int ts = c0; ts < t1; ts += CS) {
      const int tn = ts + CS;
      const int wcount = min(32, t1 - ts);
      const bool valid = lane < wcount;

      // ---- scores of this lane's token
      uint64_t accI[NSET][2], accS[NSET][2];
#pragma unroll
      for (int st = 0; st < NSET; ++st) accI[st][0] = accI[st][1] = accS[st][0] = accS[st][1] = 0ull;
      if constexpr (PROD) segment_lookups<1, 16, NSET, Lo::SETS>(accS, sw4, lutS, swap, sh, rot16);
      if constexpr (GRP)
        segment_lookups<Lo::MS, Lo::PS, NSET, Lo::SETS>(accS, kw + Lo::IBI / 4, lutS, swap, sh, rot16);
      segment_lookups<Lo::MI, PI, NSET, Lo::SETI>(accI, kw, lutI, swap, sh, rot16);
      const float n16 = half_lo(nw), r16 = TWO ? half_hi(nw) : 0.f;
      const uint4 vcur = vpar;
      // the next chunk's key bytes and value parameters, in flight during this chunk's P.V
      if (tn < t1) load_keys(tn, kw, sw4, nw, vpar);
      float sc[NH];
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        const float2 xi = up2(accI[h / 4][(h / 2) % 2]), xs = up2(accS[h / 4][(h / 2) % 2]);
        const float ai = (h & 1) ? xi.y : xi.x, as = (h & 1) ? xs.y : xs.x;
        sc[h] = TWO ? fmaf(n16, ai, r16 * as) : n16 * ai;
      }
      if (a.scores != nullptr && valid) {
#pragma unroll
        for (int h = 0; h < NH; ++h) {
          if (h < nh) {
            const int hq = gheads[h];
            a.scores[(static_cast<int64_t>(b) * a.n_q_heads + hq) * a.scores_ld + ts + lane] =
                sc[h] * a.inv_scale_log2;
          }
        }
      }
      if constexpr (HAS_V) {
        // ---- online softmax with a lazily raised reference maximum
        bool need = false;
#pragma unroll
        for (int h = 0; h < NH; ++h) need |= valid && sc[h] > m[h] + kTau;
        if (__any_sync(kFull, need)) {
#pragma unroll
          for (int h = 0; h < NH; ++h) {
            const float cm = warp_max(valid ? sc[h] : -INFINITY);
            if (cm > m[h] + kTau) {  // warp-uniform
              const float alpha = ex2(m[h] - cm);   // 0 while m = -inf
              l[h] *= alpha;
              const uint64_t al = pk2(alpha, alpha);
#pragma unroll
              for (int k = 0; k < 4; ++k) o[h][k] = mul2(o[h][k], al);
              m[h] = cm;
            }
          }
        }
        float p[NH];
#pragma unroll
        for (int h = 0; h < NH; ++h) {
          p[h] = (valid && h < nh) ? ex2(sc[h] - m[h]) : 0.f;
          l[h] += p[h];
          mx[h] = fmaxf(mx[h], valid ? sc[h] : -INFINITY);
        }
#pragma unroll
        for (int k = 0; k < NH4; ++k) {
          float q4[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) q4[i] = 4 * k + i < NH ? p[(4 * k + i) % NH] : 0.f;
          sP4[k * 32 + lane] = make_float4(q4[0], q4[1], q4[2], q4[3]);
        }
        {
          // this token's group parameters (zeros past the range: v = 0 there)
          const uint32_t pw[4] = {vcur.x, vcur.y, vcur.z, vcur.w};
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            const float mnv = half_lo(pw[g]), scv = half_hi(pw[g]);
            if constexpr (Lo::VP4)
              reinterpret_cast<float4*>(sVP)[g * kVpStride + lane] =
                  make_float4(SA * scv, SB * scv, fmaf(-SA, scv, mnv), fmaf(-SB, scv, mnv));
            else
              reinterpret_cast<float2*>(sVP)[g * kVpStride + lane] = make_float2(scv, mnv);
          }
        }
        cp_async_wait<0>();
        __syncwarp();

        // ---- P.V: token 2 jj + hw of the chunk per step, channels 8 j16 .. 8 j16 + 7.
        // Every step runs: tokens past the range carry p = 0 and v = 0 (zero parameters).
#pragma unroll 4
        for (int jj = 0; jj < 16; ++jj) {
          const int tok = 2 * jj + hw;
          uint64_t SP, CP;
          if constexpr (Lo::VP4) {
            const float4 dq = reinterpret_cast<const float4*>(sVP)[vg * kVpStride + tok];
            SP = pk2(dq.x, dq.y);
            CP = pk2(dq.z, dq.w);
          } else {
            const float2 dq = reinterpret_cast<const float2*>(sVP)[vg * kVpStride + tok];
            SP = pk2(SA * dq.x, SB * dq.x);
            CP = pk2(fmaf(-SA, dq.x, dq.y), fmaf(-SB, dq.x, dq.y));
          }
          uint64_t v[4];
          if constexpr (VB == 2) {
            const uint32_t c16 = reinterpret_cast<const uint16_t*>(sVQ + tok * 32)[j16];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const uint32_t w = c16 << (19 - 4 * k);
              v[k] = fma2(pk2(__uint_as_float(0x3f800000u | (w & 0x00180000u)),
                              __uint_as_float(0x3f800000u | (w & 0x00600000u))), SP, CP);
            }
          } else {
            const uint32_t c32 = reinterpret_cast<const uint32_t*>(sVQ + tok * 64)[j16];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const uint32_t w = k < 2 ? (c32 << (15 - 8 * k)) : (c32 >> (8 * k - 15));
              v[k] = fma2(pk2(__uint_as_float(0x3f800000u | (w & 0x00078000u)),
                              __uint_as_float(0x3f800000u | (w & 0x00780000u))), SP, CP);
            }
          }
          // p of 4 heads per 16-byte load; the (p, p) pairs are formed in registers
#pragma unroll
          for (int k4 = 0; k4 < NH4; ++k4) {
            const float4 pp = sP4[k4 * 32 + tok];
            const float pv[4] = {pp.x, pp.y, pp.z, pp.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int h = 4 * k4 + i;
              if (h < NH) {
                const uint64_t ph = pk2(pv[i], pv[i]);
#pragma unroll
                for (int k = 0; k < 4; ++k) o[h][k] = fma2(ph, v[k], o[h][k]);
              }
            }
          }
        }
        __syncwarp();
        if (tn < t1) load_codes(tn);
      }
    }
    cp_async_wait<0>();
  }
  grid_dependency_wait();  // (blocks past the longest sequence skipped the wait above)

  if constexpr (!HAS_V) return;

  // ---------------- merge the warps of this block
  __syncthreads();
  // Each warp's record per head: its reference maximum m, the lanes' sums and largest
  // logits, and the outputs of both half-warps (disjoint tokens of the same channels); the
  // block merge reduces them across lanes once per head instead of once per warp and head.
  float* sM = reinterpret_cast<float*>(smem);  // [warp][head][kWRec]
  {
    const int hw = lane >> 4, j16 = lane & 15;
#pragma unroll
    for (int h = 0; h < NH; ++h) {
      if (h < nh) {
        float* dst = sM + (warp * SL + h) * kWRec;
        if (lane == 0) dst[0] = m[h];
        dst[kWRecL + lane] = l[h];
        dst[kWRecX + lane] = mx[h];
        const float2 v0 = up2(o[h][0]), v1 = up2(o[h][1]), v2 = up2(o[h][2]), v3 = up2(o[h][3]);
        float* od = dst + kWRecO + kD * hw + 8 * j16;
        *reinterpret_cast<float4*>(od) = make_float4(v0.x, v0.y, v1.x, v1.y);
        *reinterpret_cast<float4*>(od + 4) = make_float4(v2.x, v2.y, v3.x, v3.y);
      }
    }
  }
  decode_merge<NH, SL, NT, NWp>(a, smem, &sLast, gheads, nh, b, split);
}

// Launch one instantiation (dynamic shared memory configured on first use; programmatic
// dependent launch only when asked for: right after the library's own append kernel).
template <int MB, int VB, int NH, int K, int NSET>
tq_status run_decode(const DecodeArgs& a, dim3 grid, bool pdl, cudaStream_t st) {
  constexpr int smem = Lay<MB, VB, K, NSET, NH>::total;
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
  cfg.blockDim = dim3(Shape<NSET>::threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  if (cudaLaunchKernelEx(&cfg, kern, a) != cudaSuccess) return TQ_ECUDA;
  return cudaGetLastError() == cudaSuccess ? TQ_OK : TQ_ECUDA;
}



// Two table sets where the layout fits the shared memory (and never for grouped keys, whose
// two segments already take two table kinds).
template <int MB, int VB, int K>
constexpr bool two_sets_fit() {
  if constexpr (K == kGrp) return false;
  else return Lay<MB, VB, K, 2, 8>::fits;
}

// Heads per block template: one set 2, 3 or 4, two sets 6, 7 or 8 (each P.V step works on
// every head slot of the template, so groups of 3 or 7 heads skip the empty slot).
template <int MB, int VB, int K>
tq_status run_decode_shape(const DecodeArgs& a, dim3 grid, int max_heads, bool two, bool pdl,
                           cudaStream_t st) {
  if constexpr (two_sets_fit<MB, VB, K>()) {
    if (two) {
      if (max_heads <= 6) return run_decode<MB, VB, 6, K, 2>(a, grid, pdl, st);
      if (max_heads == 7) return run_decode<MB, VB, 7, K, 2>(a, grid, pdl, st);
      return run_decode<MB, VB, 8, K, 2>(a, grid, pdl, st);
    }
  }
  if (max_heads <= 2) return run_decode<MB, VB, 2, K, 1>(a, grid, pdl, st);
  if (max_heads == 3) return run_decode<MB, VB, 3, K, 1>(a, grid, pdl, st);
  return run_decode<MB, VB, 4, K, 1>(a, grid, pdl, st);
}

// Per key kind (one translation unit each): launch the instantiation of (mb, vb).
tq_status launch_kind_prod(const DecodeArgs& a, int mb, int vb, dim3 grid, int max_heads,
                           bool two, bool pdl, cudaStream_t st);
tq_status launch_kind_mse(const DecodeArgs& a, int mb, int vb, dim3 grid, int max_heads,
                          bool two, bool pdl, cudaStream_t st);
tq_status launch_kind_grp(const DecodeArgs& a, int mb, int vb, dim3 grid, int max_heads,
                          bool two, bool pdl, cudaStream_t st);
bool two_sets_ok(int kind, int mb, int vb);

}  // namespace dec
}  // namespace tq
