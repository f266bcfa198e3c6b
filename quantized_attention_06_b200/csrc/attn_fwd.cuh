// attn_fwd.cuh - quantized attention forward on sm_100a tensor cores.
//
// Method (SageAttention): vibecrowd repo page "thu-ml--sageattention", How it
// works (INT8 QK^T, FP8/FP16 PV, two-level accumulation for PV); heatdrop review
// "2–5× attention speedups without the accuracy apology tour", The interesting
// bit (two-level accumulation inside FP8 tensor cores) and Key highlights (GQA,
// variable lengths); glossary page "SageAttention(セージアテンション)" (FlashAttention-
// compatible online softmax).
//
// CTA = one (sequence, query head, pair of 128-row Q tiles A = 2 qp and B = 2 qp + 1).
// 16 warps in four warpgroups, registers traded with setmaxnreg (128 x 56 + 128 x 88 +
// 256 x 184 = 512 x 128, the launch allocation):
//   WG0  warp 0: TMA producer (both Q tiles once, K / V tiles into rings shared by A and B)
//        warps 1 and 2: the MMA issuers of Q tiles A and B (one thread each); warp 3 idle
//          S_x(j)  = Q8_x K8(j)^T  tcgen05.mma kind::i8 -> the TMEM S buffer of tile x
//          PV_x(j) = P_x(j) V(j)   tcgen05.mma kind::f8f6f4 (e4m3) or kind::f16, A = P from
//                                  shared memory, accumulated onto O_x in FP32
//   WG1  softmax of Q tile A, WG2 of Q tile B (one thread per query row, a whole 128-key
//        row each; the running max and sum stay in the thread's registers)
//   WG3  the running-output rescale O_x = alpha O_x before PV_x(j), and the epilogue
//
// TMEM columns: S_A [0,128), S_B [128,256), O_A [256, 256 + d), O_B [384, 384 + d).  A
// softmax warpgroup loads S_x(j) into registers and frees the buffer at once (P goes to
// shared memory), so S_x(j + 1) is computed while P_x(j) is being formed.
// Every S accumulates onto the magic pattern 0x4B400000 (fp32 1.5 * 2^23), so TMEM
// returns bits(12582912 + S).  The pattern is written by the tensor core itself: before
// the INT8 steps of S(j), one kind::f16 MMA with constant operands (every A entry 512,
// every B entry 1536, K = 16, no accumulate) sets every element of the buffer to the
// fp32 value 16 * 512 * 1536 = 12582912, and the INT8 steps add S onto those bits.
//
// Per KV tile j, query row i, natural-log logits x_ij = ((S_ij q_scale_i) k_scale_j) sm_scale:
//   m'    = max(m, max_j x_ij)                      (fp64, as the definition)
//   p_j   = ps exp(x_j - m')                        (ps = 448 for e4m3 P, 1 for 16-bit P)
//   l     = l exp(m - m') + sum_j p_j   (unquantized),  P_j = round(p_j) -> smem
//   O     = O exp(m - m') + P V         (FP32 in TMEM: rescaled, then the tile's block added)
//   out   = O v_scale / l ;  lse = m' + ln(l / ps)
// p is computed in the log2 domain from fp32 operations relative to each K-scale block's
// own largest score, t = fma(S - S_max_c, c_c, nb_c) with c_c = q_scale k_scale_c sm_scale
// log2 e and nb_c = S_max_c c_c - m' log2 e + log2 ps formed in fp64 and rounded once,
// and 2^t is the hardware exponential (ex2.approx, within 2 ulp).  That p is within
// about 25 fp32 ulps of the exact value whatever the logits' magnitude.  An e4m3 code
// is an integer decided by p, so for e4m3 P every p within 32 ulps of a rounding
// midpoint is decided again in fp64 from the definition (x - m against ln(mid / 448)):
// the codes are those of the fp64 definition.  (A 16-bit P moves by one 16-bit ulp at
// such a point; its codes are taken from the fast p.)
#pragma once

#include <type_traits>

#include "sage_device.cuh"
#include "seq_table.cuh"

namespace sage {

constexpr int kAttnThreads = 512;
constexpr int kAttnLaunchRegs = 128;  // 65536 / 512
constexpr int kProducerRegs = 56;
constexpr int kCorrectionRegs = 88;
constexpr int kSoftmaxRegs = 184;
static_assert(128 * kProducerRegs + 128 * kCorrectionRegs + 256 * kSoftmaxRegs <=
                  kAttnThreads * kAttnLaunchRegs,
              "register split exceeds the launch allocation");
constexpr double kLog2E64 = 1.4426950408889634;
constexpr double kLog2_448_64 = 8.807354922057604;  // log2(448)
constexpr float kLn448 = 6.104793232414985f;         // ln(448)
constexpr int kAlphaRing = 4;                        // alpha slots between softmax and correction

// PV operand formats: P and V in e4m3 (the method), or both in the input's 16-bit type
enum : int { kPvE4m3 = 0, kPvF16 = 1, kPvBf16 = 2 };

struct AttnArgs {
  const float* q_scale;  // [Hq][T_pad/128], or [Hq][T_pad] with the per-thread granularity
  const float* k_scale;  // [Hkv][T_pad/64], or [Hkv][T_pad/32]
  const float* v_scale;  // [B][Hkv][D] (e4m3 PV only)
  void* out;
  int out_dtype;  // 0 fp16, 1 bf16, 2 fp32
  int64_t osb, osh, ost;
  float* lse;  // [Hq][T_pad] or null
  int hq, hkv, group;
  double scale;  // sm_scale (1/sqrt(d) by default), fp64 as in the definition
  int causal;
};

template <int D, int PV>
struct AttnCfg {
  static constexpr bool kExact = PV == kPvE4m3;          // codes decided at midpoints
  static constexpr int kEB = PV == kPvE4m3 ? 1 : 2;      // bytes per P / V element
  static constexpr int kKS = PV == kPvE4m3 ? 3 : 2;      // K ring stages
  static constexpr int kVS = PV == kPvE4m3 ? 3 : 2;      // V ring stages
  static constexpr int kPBufs = PV == kPvE4m3 ? 2 : 1;   // P tiles in shared memory per Q tile
  static_assert(kPBufs == 1 || kPBufs == 2, "the barrier-free buffer reuse assumes two P buffers");
  static constexpr int kTileQK = kBlkQ * D;              // bytes of one Q (or K) tile
  static constexpr int kTileV = D * kKvTile * kEB;       // bytes of one V^T tile
  static constexpr int kTileP = kBlkQ * kKvTile * kEB;   // bytes of one P tile
  static constexpr int kQOff = 0;                        // Q tiles A and B
  static constexpr int kKOff = kQOff + 2 * kTileQK;
  static constexpr int kVOff = kKOff + kKS * kTileQK;
  static constexpr int kPOff = kVOff + kVS * kTileV;     // P tiles [Q tile][buffer]
  // constant f16 operands of the prefill MMA: 128 rows x 32 B each (32-byte swizzle atoms
  // of 8 rows; every entry equal, so the layout is immaterial)
  static constexpr int kCAOff = kPOff + 2 * kPBufs * kTileP;
  static constexpr int kCBOff = kCAOff + 128 * 32;
  static constexpr int kAOff = kCBOff + 128 * 32;                  // float alpha[2][4][128]
  static constexpr int kLOff = kAOff + 2 * kAlphaRing * 128 * 4;   // float lfin[2][128]
  static constexpr int kFOff = kLOff + 2 * 128 * 4;                // double mfin[2][128]
  static constexpr int kBarOff = kFOff + 2 * 128 * 8;
  // barriers: q_full, k_full[KS], k_empty[KS], v_full[VS], v_empty[VS], then per Q tile:
  // s_full, s_free, pv_done, o_ready, epi, p_full[PB], p_free[PB], a_full[4], a_free[4];
  // and done
  static constexpr int kBarK = 1, kBarV = kBarK + 2 * kKS, kBarX = kBarV + 2 * kVS;
  static constexpr int kPerX = 5 + 2 * kPBufs + 2 * kAlphaRing;
  static constexpr int kNumBars = kBarX + 2 * kPerX + 1;
  static constexpr int kSlotOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kSlotOff + 16;
  static constexpr int kAlloc = kBytes + 1024;  // room to align the base to 1024
  static_assert(kAlloc <= 227 * 1024, "shared memory budget");
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ---- packed fp32 pair arithmetic (one instruction per two values)
using f2 = float2;
__device__ __forceinline__ f2 f2_make(float lo, float hi) { return make_float2(lo, hi); }
__device__ __forceinline__ f2 f2_fma(f2 a, f2 b, f2 c) {
  f2 d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(reinterpret_cast<uint64_t&>(d)) : "l"(reinterpret_cast<const uint64_t&>(a)), "l"(reinterpret_cast<const uint64_t&>(b)), "l"(reinterpret_cast<const uint64_t&>(c)));
  return d;
}
__device__ __forceinline__ f2 f2_add(f2 a, f2 b) {
  f2 d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(reinterpret_cast<uint64_t&>(d)) : "l"(reinterpret_cast<const uint64_t&>(a)), "l"(reinterpret_cast<const uint64_t&>(b)));
  return d;
}
__device__ __forceinline__ f2 f2_mul(f2 a, f2 b) {
  f2 d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(reinterpret_cast<uint64_t&>(d)) : "l"(reinterpret_cast<const uint64_t&>(a)), "l"(reinterpret_cast<const uint64_t&>(b)));
  return d;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Wait for this thread's TMEM loads; tying the destination registers keeps the
// compiler from using them before the wait.
__device__ __forceinline__ void tmem_wait_ld_tied(uint32_t (&r)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                 "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                 "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]),
                 "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]),
                 "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]),
                 "+r"(r[30]), "+r"(r[31])
               :
               : "memory");
}
// Registers already covered by a preceding wait: only pins them after it.
__device__ __forceinline__ void pin_regs(uint32_t (&b)[32]) {
  asm volatile(""
               : "+r"(b[0]), "+r"(b[1]), "+r"(b[2]), "+r"(b[3]), "+r"(b[4]), "+r"(b[5]),
                 "+r"(b[6]), "+r"(b[7]), "+r"(b[8]), "+r"(b[9]), "+r"(b[10]), "+r"(b[11]),
                 "+r"(b[12]), "+r"(b[13]), "+r"(b[14]), "+r"(b[15]), "+r"(b[16]), "+r"(b[17]),
                 "+r"(b[18]), "+r"(b[19]), "+r"(b[20]), "+r"(b[21]), "+r"(b[22]), "+r"(b[23]),
                 "+r"(b[24]), "+r"(b[25]), "+r"(b[26]), "+r"(b[27]), "+r"(b[28]), "+r"(b[29]),
                 "+r"(b[30]), "+r"(b[31])
               :
               : "memory");
}
__device__ __forceinline__ f2 pair_of(const uint32_t (&r)[32], int k) {
  return f2_make(__uint_as_float(r[2 * k]), __uint_as_float(r[2 * k + 1]));
}
// The S buffer is pre-filled with kMagicBits (the fp32 1.5 * 2^23 = 12582912) and the
// INT8 MMAs accumulate onto it, so TMEM returns bits(12582912 + S): an fp32 whose
// value is exactly 12582912 + S for |S| < 2^22 (|S| <= d * 127^2 here).  Those values
// are positive and ordered like S, and any difference of two is exact.
constexpr uint32_t kMagicBits = 0x4B400000u;
constexpr float kMagic = 12582912.0f;

// a[i] for a small register array and a runtime index (a chain of selects)
template <int N>
__device__ __forceinline__ float pick(const float (&a)[N], int i) {
  float v = a[0];
#pragma unroll
  for (int k = 1; k < N; ++k) v = i == k ? a[k] : v;
  return v;
}

// max of 32 magic-offset scores (masked entries hold -inf; 0 if the chunk has no valid one)
__device__ __forceinline__ float max32(const uint32_t (&r)[32]) {
  float m0 = 0.0f, m1 = 0.0f, m2 = 0.0f, m3 = 0.0f;
#pragma unroll
  for (int i = 0; i < 32; i += 8) {
    m0 = fmax3(m0, __uint_as_float(r[i]), __uint_as_float(r[i + 1]));
    m1 = fmax3(m1, __uint_as_float(r[i + 2]), __uint_as_float(r[i + 3]));
    m2 = fmax3(m2, __uint_as_float(r[i + 4]), __uint_as_float(r[i + 5]));
    m3 = fmax3(m3, __uint_as_float(r[i + 6]), __uint_as_float(r[i + 7]));
  }
  return fmax3(m0, m1, fmaxf(m2, m3));
}

// Two fp32 values -> the PV operand format, packed into 16 bits (`lo` in the low half).
template <int PV>
__device__ __forceinline__ uint32_t cvt_pair(float lo, float hi) {
  if constexpr (PV == kPvE4m3) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
  } else if constexpr (PV == kPvF16) {
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
  } else {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
  }
}

// ---- exact e4m3 decision near a rounding midpoint
// In the e4m3 normal range (p >= 2^-6) a code boundary is a value whose fp32 bits have
// their low 20 bits equal to 0x80000 (the fp32 mantissa's first three bits are kept).
// A fast p within kMidWin ulps of such a boundary is flagged.  One integer multiply-add
// tests it: key = bits(p) * 2^12 + 0x80020000 (mod 2^32) holds the low 20 bits of
// bits(p) + 0x80020 in its top 20 bits, so key < 2^18 exactly when those low 20 bits
// lie in [0x80000 - kMidWin, 0x80000 + kMidWin).  A chunk keeps the minimum key.
constexpr uint32_t kMidWin = 32;
constexpr uint32_t kDetAdd = (0x80000u + kMidWin) << 12;
constexpr uint32_t kDetLim = (2u * kMidWin) << 12;
__device__ __forceinline__ uint32_t mid_key(float p) { return __float_as_uint(p) * 4096u + kDetAdd; }

// ln((17 + 2k) / 16), k = 0..7: the log of the mantissa of the e4m3 rounding midpoint
// 2^e (1 + (2k + 1) / 16) that lies between codes with mantissas 1 + k/8 and 1 + (k+1)/8
__constant__ double kLnMidMant[8] = {
    0.06062462181643484258, 0.17185025692665922234, 0.27193371548364175883,
    0.36290549368936845314, 0.44628710262841951153, 0.52324814376454783652,
    0.59470710774669278951, 0.66139848224536500826};
constexpr double kLn2_64 = 0.69314718055994530942;
constexpr double kLn448_64 = 6.10479323241498516161;

// The value to convert for a flagged element.  The definition's p64 = 448 exp(x - m)
// with x = ((S q_scale) k_scale) sm_scale lies above the midpoint `mid` exactly when
// x - m > ln(mid / 448) = e ln 2 + ln(mantissa of mid) - ln 448, all in fp64.  The
// returned float is on that side of the midpoint, one fp32 ulp away (or the midpoint
// itself for an exact tie, which the conversion rounds to even, as the definition
// does).  Below the e4m3 normal range, or at the saturation end, the fast p is kept.
__device__ __forceinline__ float p_decided(float s, float sq, float sk, double scale, double m64,
                                           float p) {
  const uint32_t mb = ((__float_as_uint(p) + kMidWin) & 0xFFF00000u) | 0x80000u;
  const float mid = __uint_as_float(mb);
  if (!(mid >= 0x1p-6f) || mid > 448.0f) return p;
  const double thr = static_cast<double>(static_cast<int>(mb >> 23) - 127) * kLn2_64 +
                     (kLnMidMant[(mb >> 20) & 7u] - kLn448_64);
  const double x = ((static_cast<double>(s) * static_cast<double>(sq)) * static_cast<double>(sk)) * scale;
  const double dl = (x - m64) - thr;
  return dl > 0.0 ? __uint_as_float(mb + 1u) : dl < 0.0 ? __uint_as_float(mb - 1u) : mid;
}

__device__ __forceinline__ uint32_t e4m3_code(float p) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(p));
  return r & 0xFFu;
}

// Exact conversions to fp64 that stay off the conversion unit (it shares its pipe with
// the exponentials): an integer through the 2^52 + 2^31 magic, a non-negative float
// through its bits (zero and subnormal values, rare, take the conversion instruction).
__device__ __forceinline__ double int_to_f64(int v) {
  return __dsub_rn(__hiloint2double(0x43300000, static_cast<int>(static_cast<uint32_t>(v) ^ 0x80000000u)),
                   4503601774854144.0);
}
__device__ __forceinline__ double pos_f32_to_f64(float v) {
  const uint32_t u = __float_as_uint(v);
  if ((u >> 23) == 0u) {
    double d;
    asm volatile("cvt.f64.f32 %0, %1;" : "=d"(d) : "f"(v));
    return d;
  }
  return __hiloint2double(static_cast<int>((((u >> 23) + 896u) << 20) | ((u & 0x7FFFFFu) >> 3)),
                          static_cast<int>((u & 7u) << 29));
}
// S of a magic-offset score (exact: the float and the int differ by 0x4B400000 in bits)
__device__ __forceinline__ int magic_to_int(float v) {
  return static_cast<int>(__float_as_uint(v) - kMagicBits);
}

// Constants of the fast p for one K-scale block of a row, formed from fp64 factors and
// rounded once: c = q_scale k_scale sm_scale log2 e (at least the smallest normal float,
// so a dropped key's -inf stays -inf) and nb = S_max c - m' log2 e + log2 ps, S_max the
// block's largest score.  Every operation is an explicit round-to-nearest one (no
// contraction), so settle_chunk, which re-decides flagged codes, forms the same floats.
__device__ __forceinline__ double chunk_cc(double sq_sc, double sk) {
  return __dmul_rn(__dmul_rn(sq_sc, sk), kLog2E64);
}
__device__ __forceinline__ float chunk_ck(double cc) { return fmaxf(__double2float_rn(cc), 0x1p-126f); }
__device__ __forceinline__ float chunk_nb(float hmax, double cc, double ml, double log2ps) {
  return hmax > 1.0e6f
      ? __double2float_rn(__dadd_rn(__dsub_rn(__dmul_rn(int_to_f64(magic_to_int(hmax)), cc), ml), log2ps))
      : 0.0f;
}

// Byte offset of 16-byte chunk k of row `row` in a K-major int8 tile of D-byte rows
// written by TMA with the 128-byte (D = 128) or 64-byte (D = 64) swizzle.
template <int D>
__device__ __forceinline__ uint32_t swz_off(int row, int k) {
  return D == 128 ? static_cast<uint32_t>(row * 128 + ((k ^ (row & 7)) << 4))
                  : static_cast<uint32_t>(row * 64 + ((k ^ ((row >> 1) & 3)) << 4));
}

// Settling of one flagged (row r, chunk c) of a tile by a whole warp: lane i takes key 32c + i.
// S is formed again from the int8 tiles (exact), then the softmax's own fp32 steps give
// the same fast p; a p within kMidWin ulps of a midpoint is decided by p_decided and its
// code byte rewritten in the row's slot of the P tile.
// Magic-offset score of query row r and key `key` of the tile from the int8 tiles
// (-inf for a dropped key), exact.
template <int D>
__device__ __forceinline__ float score_at(uint32_t qbase, uint32_t kbase, int r, int key, bool drop) {
  int acc[4] = {0, 0, 0, 0};  // four independent dot-product chains
#pragma unroll
  for (int k = 0; k < D / 16; ++k) {
    uint32_t q4[4], k4[4];
    ld_shared16(qbase + swz_off<D>(r, k), q4);
    ld_shared16(kbase + swz_off<D>(key, k), k4);
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[e] = __dp4a(static_cast<int>(q4[e]), static_cast<int>(k4[e]), acc[e]);
  }
  const int sum = (acc[0] + acc[1]) + (acc[2] + acc[3]);
  return drop ? __uint_as_float(0xFF800000u) : kMagic + static_cast<float>(sum);
}

// kCpb = chunks per K-scale block (2: 64-key blocks, 1: 32-key blocks); `drop_sib` says
// whether this lane's key in the sibling chunk c ^ 1 is dropped.
template <int D, int kCpb>
__device__ __forceinline__ void settle_chunk(uint32_t qbase, uint32_t kbase, uint32_t pbase, int r,
                                             int c, int lane, bool drop, bool drop_sib, float sq,
                                             float sk, double scale, double m64) {
  const float sv = score_at<D>(qbase, kbase, r, 32 * c + lane, drop);
  float hm = sv;
  if (kCpb == 2) hm = fmaxf(hm, score_at<D>(qbase, kbase, r, 32 * (c ^ 1) + lane, drop_sib));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) hm = fmaxf(hm, __shfl_xor_sync(0xffffffffu, hm, o));
  hm = fmaxf(hm, 0.0f);
  const double cc = chunk_cc(__dmul_rn(static_cast<double>(sq), scale), static_cast<double>(sk));
  const float nb = chunk_nb(hm, cc, __dmul_rn(m64, kLog2E64), kLog2_448_64);
  const float p = ex2(__fmaf_rn(__fadd_rn(sv, -hm), chunk_ck(cc), nb));
  if (mid_key(p) < kDetLim) {
    const float pe = p_decided(__fsub_rn(sv, kMagic), sq, sk, scale, m64, p);
    st_shared_u8(pbase + r * 128 + ((((2 * c + (lane >> 4)) ^ (r & 7)) & 7) << 4) + (lane & 15),
                 e4m3_code(pe));
  }
}

// P for the 32 keys of chunk c of one row: t = fma(S - S_max_c, ck, nb) (the difference
// of two magic-offset floats is exact), p = 2^t, added into acc and written, in the PV
// operand format, to the row's slot of a 128-byte-swizzled K-major P tile in shared
// memory (`prow` = tile base + row * 128, `rx` = row % 8).  A dropped key holds S = -inf,
// so its t is -inf and p = 0 (ck is at least the smallest normal float).  With kExact
// (e4m3 P) the
// chunk's smallest midpoint key is returned (below kDetLim: a p to decide again).
template <int PV, bool kExact>
__device__ __forceinline__ uint32_t p_chunk(const uint32_t (&r)[32], float hmax, float ck, float nb,
                                            f2& acc, uint32_t prow, int rx, int c) {
  const f2 CK = f2_make(ck, ck), NB = f2_make(nb, nb), NH = f2_make(-hmax, -hmax);
  // one 16-byte chunk of the row at a time: 16 e4m3 codes or 8 16-bit values
  constexpr int kPerChunk = PV == kPvE4m3 ? 16 : 8;
  constexpr int kStores = 32 / kPerChunk;
  uint32_t w[kStores * 4];
  uint32_t kmin = 0xFFFFFFFFu;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const f2 t = f2_fma(f2_add(pair_of(r, i), NH), CK, NB);
    float p0 = ex2(t.x), p1 = ex2(t.y);
    acc = f2_add(acc, f2_make(p0, p1));
    if constexpr (kExact) kmin = min(kmin, min(mid_key(p0), mid_key(p1)));
    const uint32_t two = cvt_pair<PV>(p0, p1);
    if constexpr (PV == kPvE4m3) {
      if (i & 1) w[i >> 1] |= two << 16; else w[i >> 1] = two;
    } else {
      w[i] = two;
    }
  }
#pragma unroll
  for (int e = 0; e < kStores; ++e) {
    if constexpr (PV == kPvE4m3) {
      // 32 codes = 16-byte chunks 2c, 2c + 1 of the 128-byte row
      st_shared16(prow + ((((2 * c + e) ^ rx) & 7) << 4), w[4 * e], w[4 * e + 1], w[4 * e + 2],
                  w[4 * e + 3]);
    } else {
      // 64 bytes = 16-byte chunks 4c .. 4c + 3 of the 256-byte row; keys 0-63 fill
      // swizzle block 0 and keys 64-127 block 1 (128 rows x 128 B each)
      const int g = 4 * c + e;
      st_shared16(prow + ((g >> 3) * (kBlkQ * 128)) + ((((g & 7) ^ rx) & 7) << 4), w[4 * e],
                  w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
    }
  }
  return kmin;
}

template <int D, class Seq, bool kFine, int PV>
__global__ void __launch_bounds__(kAttnThreads, 1)
sage_attn_fwd_kernel(const __grid_constant__ CUtensorMap tmap_q,
                     const __grid_constant__ CUtensorMap tmap_k,
                     const __grid_constant__ CUtensorMap tmap_v,
                     const __grid_constant__ Seq seq, const __grid_constant__ AttnArgs a) {
  using L = AttnCfg<D, PV>;
  constexpr int KS = L::kKS, VS = L::kVS, PB = L::kPBufs;
  constexpr bool kExact = L::kExact;
  constexpr uint32_t kSwizzle = (D == 128) ? 2u : 4u;  // UMMA layout type: 128B / 64B swizzle
  constexpr uint32_t kSboQK = 8u * D;                  // 8 rows of D bytes
  constexpr uint32_t kIdescS = idesc_i8(128, kKvTile);
  constexpr uint32_t kIdescPV = PV == kPvE4m3 ? idesc_e4m3_f32(128, D)
                                : PV == kPvF16 ? idesc_f16_f32(128, D) : idesc_bf16_f32(128, D);
  constexpr uint32_t kIdescPre = idesc_f16_f32(128, kKvTile);
  constexpr uint32_t kColO = 256;  // S of Q tile x at columns 128 x, its O at kColO + 128 x
  constexpr double kLog2Ps = PV == kPvE4m3 ? kLog2_448_64 : 0.0;
  constexpr float kLnPs = PV == kPvE4m3 ? kLn448 : 0.0f;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + L::kBarOff;
  const uint32_t bar_q = bar0;
  auto bar_kf = [&](int s) { return bar0 + 8u * (L::kBarK + s); };
  auto bar_ke = [&](int s) { return bar0 + 8u * (L::kBarK + KS + s); };
  auto bar_vf = [&](int s) { return bar0 + 8u * (L::kBarV + s); };
  auto bar_ve = [&](int s) { return bar0 + 8u * (L::kBarV + VS + s); };
  auto bx = [&](int x, int i) { return bar0 + 8u * (L::kBarX + x * L::kPerX + i); };
  auto bar_sfull = [&](int x) { return bx(x, 0); };
  auto bar_sfree = [&](int x) { return bx(x, 1); };
  auto bar_pvdone = [&](int x) { return bx(x, 2); };
  auto bar_oready = [&](int x) { return bx(x, 3); };
  auto bar_epi = [&](int x) { return bx(x, 4); };
  auto bar_pfull = [&](int x, int s) { return bx(x, 5 + s); };
  auto bar_pfree = [&](int x, int s) { return bx(x, 5 + PB + s); };
  auto bar_afull = [&](int x, int s) { return bx(x, 5 + 2 * PB + s); };
  auto bar_afree = [&](int x, int s) { return bx(x, 5 + 2 * PB + kAlphaRing + s); };
  const uint32_t bar_done = bar0 + 8u * (L::kBarX + 2 * L::kPerX);
  float* alph = reinterpret_cast<float*>(smem + L::kAOff);     // [x][tile % 4][row]
  float* lfin = reinterpret_cast<float*>(smem + L::kLOff);     // [x][row]
  double* mfin = reinterpret_cast<double*>(smem + L::kFOff);   // [x][row]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kSlotOff);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wg = warp >> 2;

  // ---------------------------------------------------------------- work item
  // CTA = (sequence, query head, pair of 128-row Q tiles 2 qp and 2 qp + 1)
  int b, hq, qp;
  {
    int idx = blockIdx.x;
    int npair;
    if constexpr (std::is_same<Seq, SeqDense>::value) {
      b = 0;
      npair = ((seq_len(seq, 0) + kBlkQ - 1) / kBlkQ + 1) / 2;
    } else {
      int lo = 0, hi = seq.nseq - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (seq.cta[mid] <= idx) lo = mid; else hi = mid - 1;
      }
      while (lo + 1 < seq.nseq && seq.cta[lo + 1] <= idx) ++lo;
      b = lo;
      idx -= seq.cta[b];
      npair = ((seq_len(seq, b) + kBlkQ - 1) / kBlkQ + 1) / 2;
    }
    const int g = idx % a.group; idx /= a.group;
    qp = idx % npair; idx /= npair;
    const int hk = idx % a.hkv;
    if constexpr (std::is_same<Seq, SeqDense>::value) b = idx / a.hkv;
    hq = hk * a.group + g;
    if (a.causal) qp = npair - 1 - qp;  // longest rows first
  }
  const int hk = hq / a.group;
  const int n = seq_len(seq, b);
  const int off = seq_off(seq, b);
  const bool hasB = 2 * qp + 1 < (n + kBlkQ - 1) / kBlkQ;  // the second Q tile exists
  const int nX = hasB ? 2 : 1;
  // KV tiles of the pair (causal: through the last Q tile's diagonal; Q tile A then sees
  // one fully masked tile, whose P is zero)
  const int nkv = a.causal ? 2 * qp + nX : (n + kKvTile - 1) / kKvTile;

  // ---------------------------------------------------------------- set-up
  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    // a K stage is free once S of both Q tiles read it and (exact e4m3 P) their softmax
    // warps settled their flagged chunks; a V stage once both PV read it
    for (int s = 0; s < KS; ++s) {
      mbar_init(bar_kf(s), 1);
      mbar_init(bar_ke(s), nX + (kExact ? 4 * nX : 0));
    }
    for (int s = 0; s < VS; ++s) { mbar_init(bar_vf(s), 1); mbar_init(bar_ve(s), nX); }
    for (int x = 0; x < 2; ++x) {
      mbar_init(bar_sfull(x), 1);   // tcgen05.commit of S_x(j)
      mbar_init(bar_sfree(x), 4);   // the 4 softmax warps of Q tile x loaded S_x(j)
      mbar_init(bar_pvdone(x), 1);  // tcgen05.commit of PV_x(j) into O_x
      mbar_init(bar_oready(x), 4);  // the 4 correction warps rescaled O_x for tile j
      mbar_init(bar_epi(x), 4);     // the 4 softmax warps of Q tile x left l and m
      for (int s = 0; s < PB; ++s) {
        mbar_init(bar_pfull(x, s), 4);  // the 4 softmax warps wrote P_x
        mbar_init(bar_pfree(x, s), 1);  // tcgen05.commit of the PV that read it
      }
      for (int s = 0; s < kAlphaRing; ++s) {
        mbar_init(bar_afull(x, s), 4);  // the 4 softmax warps wrote the tile's alpha
        mbar_init(bar_afree(x, s), 4);  // the 4 correction warps read it
      }
    }
    mbar_init(bar_done, nX);        // a commit from each MMA issuer
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmap_q);
    tma_prefetch_desc(&tmap_k);
    tma_prefetch_desc(&tmap_v);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  {
    // prefill operands: f16 512.0 (0x6000) and 1536.0 (0x6600), two per word
    uint32_t* ca = reinterpret_cast<uint32_t*>(smem + L::kCAOff);
    uint32_t* cb = reinterpret_cast<uint32_t*>(smem + L::kCBOff);
    for (int i = threadIdx.x; i < 128 * 32 / 4; i += kAttnThreads) {
      ca[i] = 0x60006000u;
      cb[i] = 0x66006600u;
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const bool dead = watchdog_tripped();

  if (wg == 0) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kProducerRegs));
    if (warp == 0 && lane == 0 && !dead) {
      // ========================================================== TMA producer
      bool ok = true;
      mbar_arrive_expect_tx(bar_q, nX * L::kTileQK);
      const int qrow = hq * seq.t_pad + off + 2 * qp * kBlkQ;
      tma_load_2d(sbase + L::kQOff, &tmap_q, 0, qrow, bar_q);
      if (hasB) tma_load_2d(sbase + L::kQOff + L::kTileQK, &tmap_q, 0, qrow + kBlkQ, bar_q);
      int nk = 0, nv = 0;  // loads issued
      for (int j = 0; j < nkv && ok; ++j) {
        const int ks = j % KS, vs = j % VS;
        if (j >= KS) ok = mbar_wait<true>(bar_ke(ks), ((j / KS) - 1) & 1, 0x101);
        if (!ok) break;
        mbar_arrive_expect_tx(bar_kf(ks), L::kTileQK);
        tma_load_2d(sbase + L::kKOff + ks * L::kTileQK, &tmap_k, 0,
                    hk * seq.t_pad + off + j * kKvTile, bar_kf(ks));
        ++nk;
        if (j >= VS) ok = mbar_wait<true>(bar_ve(vs), ((j / VS) - 1) & 1, 0x102);
        if (!ok) break;
        mbar_arrive_expect_tx(bar_vf(vs), L::kTileV);
        if constexpr (PV == kPvE4m3) {
          tma_load_2d(sbase + L::kVOff + vs * L::kTileV, &tmap_v, off + j * kKvTile, hk * D,
                      bar_vf(vs));
        } else {
          // 16-bit V^T rows are 256 B per tile: two 128-byte-swizzled boxes of 64 keys
          const int xc = 2 * (off + j * kKvTile);
          tma_load_2d(sbase + L::kVOff + vs * L::kTileV, &tmap_v, xc, hk * D, bar_vf(vs));
          tma_load_2d(sbase + L::kVOff + vs * L::kTileV + D * 128, &tmap_v, xc + 128, hk * D,
                      bar_vf(vs));
        }
        ++nv;
      }
      // drain: the most recent load of every stage has landed before the CTA can exit
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait_sleep(bar_q, 0) && global_timer_ns() - t0 < kWaitLimitNs) {}
      for (int jj = max(0, nk - KS); jj < nk; ++jj)
        while (!mbar_try_wait_sleep(bar_kf(jj % KS), (jj / KS) & 1) &&
               global_timer_ns() - t0 < kWaitLimitNs) {}
      for (int jj = max(0, nv - VS); jj < nv; ++jj)
        while (!mbar_try_wait_sleep(bar_vf(jj % VS), (jj / VS) & 1) &&
               global_timer_ns() - t0 < kWaitLimitNs) {}
    } else if (warp >= 1 && warp <= nX && lane == 0 && !dead) {
      // ========================================================== MMA issuers
      // warp 1 issues every MMA of Q tile A, warp 2 every MMA of Q tile B.  Per KV tile j:
      // S_x(j + 1) as soon as the softmax has S_x(j) in registers, then PV_x(j), which
      // accumulates onto O_x once the correction warps have rescaled O_x for tile j.  A
      // thread's tcgen05.mma ops run in its issue order and its commits track its own
      // ops.  Descriptors differ only in their start-address field (address >> 4).
      const int x = warp - 1;
      bool ok = mbar_wait<true>(bar_q, 0, 0x201);
      const uint64_t dq = sdesc_kmajor(sbase + L::kQOff + x * L::kTileQK, kSboQK, kSwizzle);
      const uint64_t dk = sdesc_kmajor(sbase + L::kKOff, kSboQK, kSwizzle);
      const uint64_t dca = sdesc_kmajor(sbase + L::kCAOff, 256u, 6u);  // 32-byte swizzle
      const uint64_t dcb = sdesc_kmajor(sbase + L::kCBOff, 256u, 6u);
      const uint64_t dv = sdesc_kmajor(sbase + L::kVOff, 1024u, 2u);
      const uint64_t dp = sdesc_kmajor(sbase + L::kPOff + x * PB * L::kTileP, 1024u, 2u);
      const uint32_t tS = tmem + 128u * x, tO = tmem + kColO + 128u * x;
      auto issue_s = [&](int js) {
        if (!mbar_wait(bar_kf(js % KS), (js / KS) & 1, 0x203)) return false;
        tc_fence_after();
        const uint64_t bk = dk + static_cast<uint64_t>(((js % KS) * L::kTileQK) >> 4);
        mma_f16_ss(tS, dca, dcb, kIdescPre, 0u);  // every element := 12582912.0f
#pragma unroll
        for (int s = 0; s < D / 32; ++s) mma_i8_ss(tS, dq + 2u * s, bk + 2u * s, kIdescS, 1u);
        tc_commit(bar_sfull(x));
        tc_commit(bar_ke(js % KS));
        return true;
      };
      ok = ok && issue_s(0);
      for (int jp = 0; jp < nkv && ok; ++jp) {
        if (jp + 1 < nkv) {
          ok = mbar_wait(bar_sfree(x), jp & 1, 0x202) && issue_s(jp + 1);
          if (!ok) break;
        }
        // PV(jp) needs P(jp), V(jp) and, after the first tile, O rescaled for tile jp
        ok = mbar_wait(bar_pfull(x, jp % PB), (jp / PB) & 1, 0x204) &&
             mbar_wait(bar_vf(jp % VS), (jp / VS) & 1, 0x205) &&
             (jp == 0 || mbar_wait(bar_oready(x), (jp - 1) & 1, 0x206));
        if (!ok) break;
        tc_fence_after();
        const int vs = jp % VS;
        const uint64_t bv = dv + static_cast<uint64_t>((vs * L::kTileV) >> 4);
        const uint64_t ap = dp + static_cast<uint64_t>(((jp % PB) * L::kTileP) >> 4);
        if constexpr (PV == kPvE4m3) {
#pragma unroll
          for (int s = 0; s < kKvTile / 32; ++s)  // 32 keys (32 bytes) per step
            mma_f8_ss(tO, ap + 2u * s, bv + 2u * s, kIdescPV, (jp > 0 || s > 0) ? 1u : 0u);
        } else {
#pragma unroll
          for (int s = 0; s < kKvTile / 16; ++s) {  // 16 keys (32 bytes) per step
            const uint32_t blk = s >> 2, w = s & 3;  // 64-key swizzle block, step within it
            mma_f16_ss(tO, ap + ((blk * (kBlkQ * 128) + w * 32) >> 4),
                       bv + ((blk * (D * 128) + w * 32) >> 4), kIdescPV, (jp > 0 || s > 0) ? 1u : 0u);
          }
        }
        tc_commit(bar_pvdone(x));
        tc_commit(bar_ve(vs));
        tc_commit(bar_pfree(x, jp % PB));
      }
      // every MMA issued by this thread has completed before TMEM is released
      tc_commit(bar_done);
      const uint64_t t1 = global_timer_ns();
      while (!mbar_try_wait_sleep(bar_done, 0) && global_timer_ns() - t1 < kWaitLimitNs) {}
    }
  } else if (wg <= 2) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs));
    // ============================================================ softmax of Q tile x
    const int x = wg - 1;
    if (x < nX) {
      const int qt = 2 * qp + x;
      const int quarter = warp & 3;   // TMEM lane quarter this warp may access
      const int row = quarter * 32 + lane;
      const int grow = qt * kBlkQ + row;  // query index within the sequence
      const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
      const uint32_t tS = tmem + lane_base + 128u * x;
      const int rx = row & 7;
      bool ok = !dead;
      // this row's Q scale, and the K scales of the sequence
      const float sq = kFine
          ? a.q_scale[static_cast<int64_t>(hq) * seq.t_pad + off + qt * kBlkQ + row]
          : a.q_scale[static_cast<int64_t>(hq) * (seq.t_pad / kBlkQ) + off / kBlkQ + qt];
      constexpr int kblk = kFine ? kBlkKFine : kBlkK;
      const float* ksc = a.k_scale + static_cast<int64_t>(hk) * (seq.t_pad / kblk) + off / kblk;
      // K-scale blocks per tile (64-key blocks, or 32-key ones with the per-thread option)
      constexpr int kSB = kFine ? 4 : 2, kCpb = 4 / kSB;
      auto kscb = [&](int j, int bb) { return ksc[kSB * j + bb]; };
      const double sq_d = static_cast<double>(sq);
      const double sq_sc = __dmul_rn(sq_d, a.scale);  // q_scale sm_scale

      // K scales are fetched one tile ahead, off the tile's critical path
      float skn[kSB];
#pragma unroll
      for (int bb = 0; bb < kSB; ++bb) skn[bb] = kscb(0, bb);
      float l = 0.0f;            // running sum, relative to m_run
      double m_run = -INFINITY;  // running max of the logits (fp64, as the definition)
      for (int j = 0; j < nkv && ok; ++j) {
        float sk[kSB];
#pragma unroll
        for (int bb = 0; bb < kSB; ++bb) {
          sk[bb] = skn[bb];
          skn[bb] = j + 1 < nkv ? kscb(j + 1, bb) : 0.0f;
        }
        const bool masked = (a.causal && j >= qt) || (j + 1) * kKvTile > n;
        const int kv0 = j * kKvTile;  // first key of the tile
        auto dropped = [&](int key) { return key >= n || (a.causal && key > grow); };
        ok = __all_sync(0xffffffffu, mbar_wait(bar_sfull(x), j & 1, 0x301 + x));
        if (!ok) break;
        tc_fence_after();

        uint32_t s[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(tS + 32u * c, s[c]);
        tmem_wait_ld_tied(s[0]);
        pin_regs(s[1]);
        pin_regs(s[2]);
        pin_regs(s[3]);
        // S is in registers: the buffer may take S(j + 1)
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_sfree(x));

        if (masked) {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              if (dropped(kv0 + 32 * c + i)) s[c][i] = 0xFF800000u;  // -inf
            }
          }
        }
        // each K-scale block's largest score; the tile's max logit x = ((S q_scale) k_scale)
        // sm_scale in fp64 (x is monotone in S within a block, so this is max_j x_j)
        float hb[kSB];
        double skd[kSB];
        double mt = -INFINITY;
#pragma unroll
        for (int bb = 0; bb < kSB; ++bb) {
          hb[bb] = kCpb == 2 ? fmaxf(max32(s[2 * bb]), max32(s[2 * bb + 1])) : max32(s[bb]);
          skd[bb] = pos_f32_to_f64(sk[bb]);
          if (hb[bb] > 1.0e6f) {
            const double xm = __dmul_rn(__dmul_rn(__dmul_rn(int_to_f64(magic_to_int(hb[bb])), sq_d), skd[bb]), a.scale);
            mt = fmax(mt, xm);
          }
        }
        const double m_new = fmax(m_run, mt);
        // alpha = e^(m - m') rescales l here and O in the correction warps (slot j % 4)
        const float alpha = ex2(static_cast<float>((m_run - m_new) * kLog2E64));
        // With two P buffers no wait is needed before reusing alpha slot j % 4 or P buffer
        // j % 2: the commit that completed S(j) covers every earlier MMA of this Q tile's
        // issuer, PV(j - 2) among them, and PV(j - 2) was issued only after the correction
        // warps had read alpha(j - 2) (they read the alphas in tile order).  With one P
        // buffer (16-bit P) PV(j - 1) is issued after S(j), so both waits stay.
        if (PB == 1 && j >= kAlphaRing) {
          const int jo = j - kAlphaRing;
          ok = __all_sync(0xffffffffu, mbar_wait(bar_afree(x, jo % kAlphaRing), (jo / kAlphaRing) & 1, 0x305 + x));
          if (!ok) break;
        }
        alph[(x * kAlphaRing + j % kAlphaRing) * 128 + row] = alpha;
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_afull(x, j % kAlphaRing));
        // per K-scale block: c = q_scale k_scale sm_scale log2 e and
        // nb = S_max c - m' log2 e + log2 ps, in fp64, each rounded once (formed while the
        // P buffer may still be in use where registers allow: with e4m3 P)
        float ckb[kSB], nbb[kSB];
        if constexpr (PV == kPvE4m3) {
          const double ml = __dmul_rn(m_new, kLog2E64);
#pragma unroll
          for (int bb = 0; bb < kSB; ++bb) {
            const double cc = chunk_cc(sq_sc, skd[bb]);
            ckb[bb] = chunk_ck(cc);
            nbb[bb] = chunk_nb(hb[bb], cc, ml, kLog2Ps);
          }
        }
        // the P buffer of tile j was last read by PV(j - PB)
        const int pb = j % PB;
        if (PB == 1 && j >= PB) {
          const int jo = j - PB;
          ok = __all_sync(0xffffffffu, mbar_wait(bar_pfree(x, jo % PB), (jo / PB) & 1, 0x307 + x));
          if (!ok) break;
        }
        if constexpr (PV != kPvE4m3) {
          const double ml = __dmul_rn(m_new, kLog2E64);
#pragma unroll
          for (int bb = 0; bb < kSB; ++bb) {
            const double cc = chunk_cc(sq_sc, skd[bb]);
            ckb[bb] = chunk_ck(cc);
            nbb[bb] = chunk_nb(hb[bb], cc, ml, kLog2Ps);
          }
        }
        const uint32_t ptile = sbase + L::kPOff + (x * PB + pb) * L::kTileP;
        const uint32_t prow = ptile + row * 128;
        f2 acc = make_float2(0.0f, 0.0f);
        uint32_t flag = 0u;  // lane c < 4: which rows of this warp have a flagged p in chunk c
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint32_t kmin = p_chunk<PV, kExact>(s[c], hb[c / kCpb], ckb[c / kCpb], nbb[c / kCpb], acc, prow, rx, c);
          if constexpr (kExact) {
            const uint32_t bm = __ballot_sync(0xffffffffu, kmin < kDetLim);
            flag = lane == c ? bm : flag;
          }
        }
        if constexpr (kExact) {
          // Rare: chunks holding a p near an e4m3 rounding midpoint.  The warp settles them
          // together (one key per lane, settle_chunk) before P(j) is published; then it
          // releases K(j).
          uint32_t nzc = __ballot_sync(0xffffffffu, lane < 4 && flag != 0u);
          while (nzc != 0u) {
            const int c = __ffs(nzc) - 1;
            nzc &= nzc - 1u;
            uint32_t bm = __shfl_sync(0xffffffffu, flag, c);
            const float skc = pick(sk, c / kCpb);
            const int key = kv0 + 32 * c + lane, key2 = kv0 + 32 * (c ^ 1) + lane;
            while (bm != 0u) {
              const int rl = __ffs(bm) - 1;
              bm &= bm - 1u;
              const int r = quarter * 32 + rl;
              const int gr = qt * kBlkQ + r;
              const double m64 = __shfl_sync(0xffffffffu, m_new, rl);
              const float sqr = kFine ? __shfl_sync(0xffffffffu, sq, rl) : sq;
              settle_chunk<D, kCpb>(sbase + L::kQOff + x * L::kTileQK,
                                    sbase + L::kKOff + (j % KS) * L::kTileQK, ptile, r, c, lane,
                                    key >= n || (a.causal && key > gr), key2 >= n || (a.causal && key2 > gr),
                                    sqr, skc, a.scale, m64);
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(bar_ke(j % KS));
        }
        l = l * alpha + (acc.x + acc.y);
        m_run = m_new;
        fence_proxy_async_smem();  // P stores -> visible to the tensor core
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_pfull(x, pb));
      }
      // hand the row's sum, and the max it is relative to, to the epilogue
      lfin[x * 128 + row] = l;
      mfin[x * 128 + row] = m_run;
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_epi(x));
    }
  } else {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kCorrectionRegs));
    // ============================================================ running-output rescale
    // O_x = alpha O_x in FP32 before PV_x(j) adds the tile's P V block onto it; skipped
    // by a warp whose 32 rows all keep their max (alpha = 1)
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    bool ok = !dead;

    for (int j = 0; j < nkv && ok; ++j) {
      for (int x = 0; x < nX && ok; ++x) {
        const int sa = j % kAlphaRing;
        ok = __all_sync(0xffffffffu, mbar_wait(bar_afull(x, sa), (j / kAlphaRing) & 1, 0x401 + x));
        if (!ok) break;
        const float al = alph[(x * kAlphaRing + sa) * 128 + row];
        __syncwarp();
        if (PB == 1 && lane == 0) mbar_arrive(bar_afree(x, sa));
        if (j == 0) continue;  // PV_x(0) starts O_x afresh
        // O_x holds PV_x(j - 1) complete before it is rescaled
        ok = __all_sync(0xffffffffu, mbar_wait(bar_pvdone(x), (j - 1) & 1, 0x403 + x));
        if (!ok) break;
        tc_fence_after();
        if (__any_sync(0xffffffffu, al != 1.0f)) {
          const uint32_t tO = tmem + lane_base + kColO + 128u * x;
          const f2 AL = make_float2(al, al);
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t ro[32];
            tmem_ld32(tO + 32u * c, ro);
            tmem_wait_ld_tied(ro);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const f2 o = f2_mul(pair_of(ro, i), AL);
              ro[2 * i] = __float_as_uint(o.x);
              ro[2 * i + 1] = __float_as_uint(o.y);
            }
            tmem_st32(tO + 32u * c, ro);
          }
          tmem_wait_st();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_oready(x));
      }
    }

    // ---------------------------------------------------------------- epilogue
    const float* vs = a.v_scale + (static_cast<int64_t>(b) * a.hkv + hk) * D;
    for (int x = 0; x < nX && ok; ++x) {
      ok = __all_sync(0xffffffffu, mbar_wait<true>(bar_pvdone(x), (nkv - 1) & 1, 0x405 + x)) &&
           __all_sync(0xffffffffu, mbar_wait<true>(bar_epi(x), 0, 0x407 + x));
      if (!ok) break;
      tc_fence_after();
      const int grow = (2 * qp + x) * kBlkQ + row;
      const double m = mfin[x * 128 + row];
      const float l = lfin[x * 128 + row];
      const float inv_l = 1.0f / l;
      const uint32_t tO = tmem + lane_base + kColO + 128u * x;
      const int64_t orow =
          seq_base(seq, b, a.osb, a.ost) + hq * a.osh + static_cast<int64_t>(grow) * a.ost;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t ro[32];
        tmem_ld32(tO + 32u * c, ro);
        tmem_wait_ld_tied(ro);
        if (grow < n) {
          float v[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float sv = PV == kPvE4m3 ? vs[32 * c + i] : 1.0f;
            v[i] = __uint_as_float(ro[i]) * sv * inv_l;
          }
          if (a.out_dtype == 2) {
            float* dst = reinterpret_cast<float*>(a.out) + orow + 32 * c;
#pragma unroll
            for (int i = 0; i < 32; i += 4)
              *reinterpret_cast<float4*>(dst + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
          } else if (a.out_dtype == 1) {
            __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(a.out) + orow + 32 * c;
#pragma unroll
            for (int i = 0; i < 32; i += 8) {
              __align__(16) __nv_bfloat16 h8[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) h8[e] = __float2bfloat16_rn(v[i + e]);
              *reinterpret_cast<uint4*>(dst + i) = *reinterpret_cast<const uint4*>(h8);
            }
          } else {
            __half* dst = reinterpret_cast<__half*>(a.out) + orow + 32 * c;
#pragma unroll
            for (int i = 0; i < 32; i += 8) {
              __align__(16) __half h8[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) h8[e] = __float2half_rn(v[i + e]);
              *reinterpret_cast<uint4*>(dst + i) = *reinterpret_cast<const uint4*>(h8);
            }
          }
        }
      }
      if (a.lse != nullptr && grow < n)
        a.lse[static_cast<int64_t>(hq) * seq.t_pad + off + grow] =
            static_cast<float>(m) + (logf(l) - kLnPs);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace sage
