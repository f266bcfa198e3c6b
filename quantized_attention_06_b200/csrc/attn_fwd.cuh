// attn_fwd.cuh - quantized attention forward on sm_100a tensor cores.
//
// Method (SageAttention): vibecrowd repo page "thu-ml--sageattention", How it
// works (INT8 QK^T, FP8 PV, two-level accumulation for PV); heatdrop review
// "2–5× attention speedups without the accuracy apology tour", The interesting
// bit (two-level accumulation inside FP8 tensor cores) and Key highlights (GQA,
// variable lengths); glossary page "SageAttention(セージアテンション)" (FlashAttention-
// compatible online softmax).
//
// CTA = one (sequence, query head, 128-row Q tile).  16 warps in four warpgroups,
// registers traded with setmaxnreg (128 x 40 + 128 x 88 + 256 x 192 = 512 x 128,
// the launch allocation):
//   WG0  warp 0: TMA producer (Q once, K / V tiles into 3-stage rings)
//        warp 1: TMEM owner and MMA issuer (one thread); warps 2-3 idle
//          S(j)  = Q8 K8(j)^T   tcgen05.mma kind::i8 -> TMEM buffer j % 2 (double-buffered)
//          PV(j) = P8(j) V8(j)  tcgen05.mma kind::f8f6f4, A = P8 from TMEM -> fresh FP32
//   WG1  softmax for keys 0-63 of every KV tile   (one thread per query row)
//   WG2  softmax for keys 64-127 of every KV tile (one thread per query row)
//   WG3  two-level accumulation O = alpha O + PV(j) held in TMEM, and the epilogue
// The two softmax warps of a lane quarter exchange their half-row maxima through
// shared memory (one mbarrier per quarter and buffer), so both take the same running max.
//
// TMEM columns: [0,128) S buffer 0, [128,256) S buffer 1, [256,256+d) PV(j),
// [384,384+d) running O.  In S buffer b, P8 of keys 0-63 goes to columns 0-15 and
// of keys 64-127 to columns 64-79 (4 e4m3 per column), each over columns its own
// softmax warps have already read; the PV MMA takes one TMEM address per 32-key step.
// Every S accumulates onto the magic pattern 0x4B400000 (fp32 1.5 * 2^23), so TMEM
// returns bits(12582912 + S).  The pattern is written by the tensor core itself: before
// the INT8 steps of S(j), one kind::f16 MMA with constant operands (every A entry 512,
// every B entry 1536, K = 16, no accumulate) sets every element of the buffer to the
// fp32 value 16 * 512 * 1536 = 12582912, and the INT8 steps add S onto those bits as
// int32.  A buffer is free for S(j + 2) once the softmax warps have read S(j) and
// written P8(j), and PV(j) has read P8(j).
//
// Per KV tile j, query row i (log2 domain, u = x * log2 e):
//   u_j   = S_ij * (q_scale * k_scale_j * sm_scale * log2 e)
//   m'    = max(m, max_j u_j);  alpha = 2^(m - m')
//   p_j   = 2^(u_j - m' + log2 448)   (= 448 * exp(x_j - x_max'), exp2_poly below)
//   l     = l * alpha + sum_j p_j     (unquantized), P8_j = e4m3(p_j) -> TMEM
//   O     = O * alpha + PV_blk        (PV_blk = P8 V8 in FP32, fresh each tile)
//   out   = O * v_scale / l ;  lse = m' ln 2 + ln(l / 448)
#pragma once

#include <type_traits>

#include "sage_device.cuh"
#include "seq_table.cuh"

namespace sage {

constexpr int kAttnThreads = 512;
constexpr int kAttnLaunchRegs = 128;  // 65536 / 512
constexpr int kProducerRegs = 40;
constexpr int kCorrectionRegs = 88;
constexpr int kSoftmaxRegs = 192;
static_assert(128 * kProducerRegs + 128 * kCorrectionRegs + 256 * kSoftmaxRegs <=
                  kAttnThreads * kAttnLaunchRegs,
              "register split exceeds the launch allocation");
constexpr int kKStages = 3;
constexpr int kVStages = 3;
constexpr float kLog2E = 1.4426950408889634f;
constexpr float kLog2_448 = 8.807354922057604f;  // log2(448)
constexpr float kLn448 = 6.104793232414985f;     // ln(448)

struct AttnArgs {
  const float* q_scale;  // [Hq][T_pad/128]
  const float* k_scale;  // [Hkv][T_pad/64]
  const float* v_scale;  // [B][Hkv][D]
  void* out;
  int out_dtype;  // 0 fp16, 1 bf16, 2 fp32
  int64_t osb, osh, ost;
  float* lse;  // [Hq][T_pad] or null
  int hq, hkv, group;
  float scale_log2;  // sm_scale * log2(e)
  int causal;
  int fine;  // per-thread granularity: q_scale per token, k_scale per 32-token block
};

template <int D>
struct AttnSmem {
  static constexpr int kTileQ = kBlkQ * D;    // bytes of one Q (or K) tile
  static constexpr int kTileV = D * kKvTile;  // bytes of one V^T tile
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQOff + kTileQ;
  static constexpr int kVOff = kKOff + kKStages * kTileQ;
  static constexpr int kXOff = kVOff + kVStages * kTileV;  // float xchg[2][2][128]
  static constexpr int kAOff = kXOff + 2 * 2 * 128 * 4;    // float alpha[2][128]
  static constexpr int kLOff = kAOff + 2 * 128 * 4;        // float lfin[2][128], mfin[128]
  // constant f16 operands of the prefill MMA: 128 rows x 128 B each (128-byte swizzle
  // atoms; every entry equal, so the layout is immaterial)
  static constexpr int kCAOff = ((kLOff + 3 * 128 * 4) + 1023) / 1024 * 1024;
  static constexpr int kCBOff = kCAOff + 128 * 128;
  static constexpr int kBarOff = kCBOff + 128 * 128;
  // barriers: q_full, k_full[3], k_empty[3], v_full[3], v_empty[3], s_full[2], s_free[2],
  // p_full[2], pv_full, pv_free, epi, mma_done, xchg[2][4] -> 31
  static constexpr int kNumBars = 31;
  static constexpr int kSlotOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kSlotOff + 16;
  static constexpr int kAlloc = kBytes + 1024;  // room to align the base to 1024
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^t in plain IEEE fp32 operations, so that the P8 code it decides can be
// reproduced exactly on any host: Cody-Waite split t = n + f with n = rint(t)
// taken by magic-number rounding (r = t + 1.5 * 2^23, bits(r) = 0x4B400000 + n)
// and f = t - (r - 1.5 * 2^23) in [-1/2, 1/2], a degree-2 polynomial for 2^f
// (coefficients fitted for minimal relative error with the constant term fixed at
// 1, so integer t gives exact powers of two; max relative error 1.97e-3, well below
// the e4m3 step of P, which is 6.25% to 12.5%), and n added to the exponent field,
// clamped below at -125 so the result stays a normal number.
constexpr float kExp2C1 = 0.702944696f;  // 0x3f33f42f
constexpr float kExp2C2 = 0.239866376f;  // 0x3e759f88
constexpr int kExpClampBits = 0x4B400000 - 125;
__device__ __forceinline__ float exp2_poly(float t) {
  const float r = __fadd_rn(t, 12582912.0f);
  const float f = __fsub_rn(t, __fsub_rn(r, 12582912.0f));
  float p = __fmaf_rn(kExp2C2, f, kExp2C1);
  p = __fmaf_rn(p, f, 1.0f);
  const int rb = max(__float_as_int(r), kExpClampBits);
  return __int_as_float(__float_as_int(p) + rb * (1 << 23));
}

// ---- packed fp32 pair arithmetic (one instruction per two values); element 0 of a
// pair is .x, handed to the f32x2 instructions as the low half of a 64-bit register.
using f2 = float2;
__device__ __forceinline__ f2 f2_make(float lo, float hi) { return make_float2(lo, hi); }
__device__ __forceinline__ float f2_lo(f2 a) { return a.x; }
__device__ __forceinline__ float f2_hi(f2 a) { return a.y; }
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
__device__ __forceinline__ void tmem_wait_ld_tied(uint32_t (&a)[32], uint32_t (&b)[32]) {
  tmem_wait_ld_tied(a);
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
// The S region is pre-filled with kMagicBits (the fp32 1.5 * 2^23 = 12582912) and the
// INT8 MMAs accumulate onto it, so TMEM returns bits(12582912 + S): an fp32 whose
// value is exactly 12582912 + S for |S| < 2^22 (|S| <= d * 127^2 here).  Those values
// are positive and ordered like S, and S itself is one exact subtraction away.
constexpr uint32_t kMagicBits = 0x4B400000u;
constexpr float kMagic = 12582912.0f;

// max of acc and 32 magic-offset scores (masked entries hold 0, below every valid value)
__device__ __forceinline__ float max32(const uint32_t (&r)[32], float acc) {
  float m0 = acc, m1 = 0.0f, m2 = 0.0f, m3 = 0.0f;
#pragma unroll
  for (int i = 0; i < 32; i += 8) {
    m0 = fmax3(m0, __uint_as_float(r[i]), __uint_as_float(r[i + 1]));
    m1 = fmax3(m1, __uint_as_float(r[i + 2]), __uint_as_float(r[i + 3]));
    m2 = fmax3(m2, __uint_as_float(r[i + 4]), __uint_as_float(r[i + 5]));
    m3 = fmax3(m3, __uint_as_float(r[i + 6]), __uint_as_float(r[i + 7]));
  }
  return fmax3(m0, m1, fmaxf(m2, m3));
}

// P for 32 keys of one 64-key half: S = (12582912 + S) - 12582912 (exact),
// t = fma(S, ck, log2 448 - m'), p = exp2_poly(t) evaluated two values per
// instruction (the same fp32 operations as exp2_poly).  Returns the e4m3 codes
// packed four per word and adds p into acc.  With kMasked, key i is kept only
// when bit i of `keep` is set; dropped keys get p = 0.
template <bool kMasked>
__device__ __forceinline__ void p8_chunk(const uint32_t (&r)[32], float ck, float nb, f2& acc,
                                         uint32_t (&w)[8], uint32_t keep) {
  const f2 CK = f2_make(ck, ck), NB = f2_make(nb, nb);
  const f2 M = f2_make(kMagic, kMagic), NM = f2_make(-kMagic, -kMagic);
  const f2 NEG1 = f2_make(-1.0f, -1.0f), ONE = f2_make(1.0f, 1.0f);
  const f2 C1 = f2_make(kExp2C1, kExp2C1), C2 = f2_make(kExp2C2, kExp2C2);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    f2 pp[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const f2 t = f2_fma(f2_add(pair_of(r, 2 * i + h), NM), CK, NB);
      const f2 rr = f2_add(t, M);
      const f2 f = f2_fma(f2_add(rr, NM), NEG1, t);
      f2 p = f2_fma(C2, f, C1);
      p = f2_fma(p, f, ONE);
      // bits(rr) = 0x4B400000 + n: max() clamps n at -125, and bits << 23 is n << 23
      // modulo 2^32
      uint32_t lo = __float_as_uint(p.x) + (static_cast<uint32_t>(max(__float_as_int(rr.x), kExpClampBits)) << 23);
      uint32_t hi = __float_as_uint(p.y) + (static_cast<uint32_t>(max(__float_as_int(rr.y), kExpClampBits)) << 23);
      if (kMasked) {
        const int e = 4 * i + 2 * h;
        lo = ((keep >> e) & 1u) ? lo : 0u;
        hi = ((keep >> (e + 1)) & 1u) ? hi : 0u;
      }
      pp[h] = f2_make(__uint_as_float(lo), __uint_as_float(hi));
    }
    acc = f2_add(acc, f2_add(pp[0], pp[1]));
    w[i] = e4m3x2(f2_lo(pp[0]), f2_hi(pp[0])) | (e4m3x2(f2_lo(pp[1]), f2_hi(pp[1])) << 16);
  }
}

template <int D, class Seq>
__global__ void __launch_bounds__(kAttnThreads, 1)
sage_attn_fwd_kernel(const __grid_constant__ CUtensorMap tmap_q,
                     const __grid_constant__ CUtensorMap tmap_k,
                     const __grid_constant__ CUtensorMap tmap_v,
                     const __grid_constant__ Seq seq, const __grid_constant__ AttnArgs a) {
  using L = AttnSmem<D>;
  constexpr uint32_t kSwizzle = (D == 128) ? 2u : 4u;  // UMMA layout type: 128B / 64B swizzle
  constexpr uint32_t kSboQK = 8u * D;                  // 8 rows of D bytes
  constexpr uint32_t kIdescS = idesc_i8(128, kKvTile);
  constexpr uint32_t kIdescPV = idesc_e4m3_f32(128, D);
  constexpr uint32_t kIdescPre = idesc_f16_f32(128, kKvTile);
  constexpr uint32_t kColPV = 256, kColO = 384;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + L::kBarOff;
  auto bar_q = [&]() { return bar0; };
  auto bar_kf = [&](int s) { return bar0 + 8u * (1 + s); };
  auto bar_ke = [&](int s) { return bar0 + 8u * (4 + s); };
  auto bar_vf = [&](int s) { return bar0 + 8u * (7 + s); };
  auto bar_ve = [&](int s) { return bar0 + 8u * (10 + s); };
  auto bar_sfull = [&](int b) { return bar0 + 8u * (13 + b); };
  auto bar_sfree = [&](int b) { return bar0 + 8u * (15 + b); };
  auto bar_pfull = [&](int b) { return bar0 + 8u * (17 + b); };
  const uint32_t bar_pvfull = bar0 + 8u * 19;
  const uint32_t bar_pvfree = bar0 + 8u * 20;
  const uint32_t bar_epi = bar0 + 8u * 21;
  const uint32_t bar_done = bar0 + 8u * 22;
  // the two softmax warps of lane quarter q swap half-row maxima through xchg
  auto bar_xchg = [&](int buf, int q) { return bar0 + 8u * (23 + 4 * buf + q); };
  float* xchg = reinterpret_cast<float*>(smem + L::kXOff);  // [buffer][half][row]
  float* alph = reinterpret_cast<float*>(smem + L::kAOff);  // [buffer][row]
  float* lfin = reinterpret_cast<float*>(smem + L::kLOff);  // [half][row], then mfin[row]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kSlotOff);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wg = warp >> 2;

  // ---------------------------------------------------------------- work item
  int b, hq, qt;
  {
    int idx = blockIdx.x;
    int ntiles;
    if constexpr (std::is_same<Seq, SeqDense>::value) {
      b = 0;
      ntiles = (seq_len(seq, 0) + kBlkQ - 1) / kBlkQ;
    } else {
      int lo = 0, hi = seq.nseq - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (seq.cta[mid] <= idx) lo = mid; else hi = mid - 1;
      }
      while (lo + 1 < seq.nseq && seq.cta[lo + 1] <= idx) ++lo;
      b = lo;
      idx -= seq.cta[b];
      ntiles = (seq_len(seq, b) + kBlkQ - 1) / kBlkQ;
    }
    const int g = idx % a.group; idx /= a.group;
    qt = idx % ntiles; idx /= ntiles;
    const int hk = idx % a.hkv;
    if constexpr (std::is_same<Seq, SeqDense>::value) b = idx / a.hkv;
    hq = hk * a.group + g;
    if (a.causal) qt = ntiles - 1 - qt;  // longest rows first
  }
  const int hk = hq / a.group;
  const int n = seq_len(seq, b);
  const int off = seq_off(seq, b);
  const int nkv = a.causal ? qt + 1 : (n + kKvTile - 1) / kKvTile;

  // ---------------------------------------------------------------- set-up
  if (threadIdx.x == 0) {
    mbar_init(bar_q(), 1);
    for (int s = 0; s < kKStages; ++s) { mbar_init(bar_kf(s), 1); mbar_init(bar_ke(s), 1); }
    for (int s = 0; s < kVStages; ++s) { mbar_init(bar_vf(s), 1); mbar_init(bar_ve(s), 1); }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar_sfull(s), 1);
      mbar_init(bar_sfree(s), 12);  // 8 softmax warps + 4 correction warps re-arm buffer s
      mbar_init(bar_pfull(s), 8);   // 8 softmax warps wrote P (and alpha) into buffer s
    }
    mbar_init(bar_pvfull, 1);
    mbar_init(bar_pvfree, 4);
    mbar_init(bar_epi, 8);
    mbar_init(bar_done, 1);
    for (int i = 0; i < 8; ++i) mbar_init(bar_xchg(i >> 2, i & 3), 2);
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
    for (int i = threadIdx.x; i < 128 * 128 / 4; i += kAttnThreads) {
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
      mbar_arrive_expect_tx(bar_q(), L::kTileQ);
      tma_load_2d(sbase + L::kQOff, &tmap_q, 0, hq * seq.t_pad + off + qt * kBlkQ, bar_q());
      int nk = 0, nv = 0;  // loads issued
      for (int j = 0; j < nkv && ok; ++j) {
        const int ks = j % kKStages, vs = j % kVStages;
        if (j >= kKStages) ok = mbar_wait<true>(bar_ke(ks), ((j / kKStages) - 1) & 1, 0x101);
        if (!ok) break;
        mbar_arrive_expect_tx(bar_kf(ks), L::kTileQ);
        tma_load_2d(sbase + L::kKOff + ks * L::kTileQ, &tmap_k, 0,
                    hk * seq.t_pad + off + j * kKvTile, bar_kf(ks));
        ++nk;
        if (j >= kVStages) ok = mbar_wait<true>(bar_ve(vs), ((j / kVStages) - 1) & 1, 0x102);
        if (!ok) break;
        mbar_arrive_expect_tx(bar_vf(vs), L::kTileV);
        tma_load_2d(sbase + L::kVOff + vs * L::kTileV, &tmap_v, off + j * kKvTile, hk * D,
                    bar_vf(vs));
        ++nv;
      }
      // drain: the most recent load of every stage has landed before the CTA can exit
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait_sleep(bar_q(), 0) && global_timer_ns() - t0 < kWaitLimitNs) {}
      for (int jj = max(0, nk - kKStages); jj < nk; ++jj)
        while (!mbar_try_wait_sleep(bar_kf(jj % kKStages), (jj / kKStages) & 1) &&
               global_timer_ns() - t0 < kWaitLimitNs) {}
      for (int jj = max(0, nv - kVStages); jj < nv; ++jj)
        while (!mbar_try_wait_sleep(bar_vf(jj % kVStages), (jj / kVStages) & 1) &&
               global_timer_ns() - t0 < kWaitLimitNs) {}
    } else if (warp == 1 && lane == 0 && !dead) {
      // ========================================================== MMA issuer
      // descriptors differ only in their start-address field (bits 0-13, address >> 4)
      const uint64_t dq = sdesc_kmajor(sbase + L::kQOff, kSboQK, kSwizzle);
      const uint64_t dk = sdesc_kmajor(sbase + L::kKOff, kSboQK, kSwizzle);
      const uint64_t dv = sdesc_kmajor(sbase + L::kVOff, 1024u, 2u);
      const uint64_t dca = sdesc_kmajor(sbase + L::kCAOff, 1024u, 2u);
      const uint64_t dcb = sdesc_kmajor(sbase + L::kCBOff, 1024u, 2u);
      auto issue_s = [&](int js) {  // S(js) = Q8 K8(js)^T onto the armed buffer js % 2
        const int ks = js % kKStages;
        const uint64_t bk = dk + static_cast<uint64_t>((ks * L::kTileQ) >> 4);
        const uint32_t d_tmem = tmem + 128u * (js & 1);
        mma_f16_ss(d_tmem, dca, dcb, kIdescPre, 0u);  // every element := 12582912.0f
#pragma unroll
        for (int s = 0; s < D / 32; ++s) mma_i8_ss(d_tmem, dq + 2u * s, bk + 2u * s, kIdescS, 1u);
        tc_commit(bar_sfull(js & 1));
        tc_commit(bar_ke(ks));
      };
      auto issue_pv = [&](int j) {  // PV(j) = P8(j) V8(j) into a fresh FP32 accumulator
        const int vs = j % kVStages;
        const uint64_t bv = dv + static_cast<uint64_t>((vs * L::kTileV) >> 4);
        const uint32_t p_tmem = tmem + 128u * (j & 1);
#pragma unroll
        for (int s = 0; s < kKvTile / 32; ++s) {
          // keys 32s..32s+31: P8 columns 0, 8 (first half) and 64, 72 (second half)
          const uint32_t a_col = (s < 2) ? 8u * s : 64u + 8u * (s - 2);
          mma_f8_ts(tmem + kColPV, p_tmem + a_col, bv + 2u * s, kIdescPV, s > 0 ? 1u : 0u);
        }
        tc_commit(bar_pvfull);
        tc_commit(bar_ve(vs));
      };
      bool ok = mbar_wait<true>(bar_q(), 0, 0x201);
      for (int js = 0; js < 2 && js < nkv && ok; ++js) {
        ok = mbar_wait<true>(bar_kf(js % kKStages), (js / kKStages) & 1, 0x202) &&
             mbar_wait<true>(bar_sfree(js & 1), 0, 0x203);
        if (!ok) break;
        tc_fence_after();
        issue_s(js);
      }
      for (int j = 0; j < nkv && ok; ++j) {
        ok = mbar_wait<true>(bar_pfull(j & 1), (j >> 1) & 1, 0x204) &&
             mbar_wait<true>(bar_vf(j % kVStages), (j / kVStages) & 1, 0x205) &&
             (j == 0 || mbar_wait<true>(bar_pvfree, (j - 1) & 1, 0x206));
        if (!ok) break;
        tc_fence_after();
        issue_pv(j);
        const int js = j + 2;
        if (js < nkv) {
          ok = mbar_wait<true>(bar_kf(js % kKStages), (js / kKStages) & 1, 0x207) &&
               mbar_wait<true>(bar_sfree(js & 1), (js >> 1) & 1, 0x208);
          if (!ok) break;
          tc_fence_after();
          issue_s(js);
        }
      }
      // every MMA issued by this thread has completed before TMEM is released
      tc_commit(bar_done);
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait_sleep(bar_done, 0) && global_timer_ns() - t0 < kWaitLimitNs) {}
    }
  } else if (wg <= 2) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs));
    // ============================================================ softmax (one 64-key half)
    const int h = wg - 1;           // 0: keys 0-63 of each KV tile, 1: keys 64-127
    const int quarter = warp & 3;   // TMEM lane quarter this warp may access
    const int row = quarter * 32 + lane;
    const int grow = qt * kBlkQ + row;  // query index within the sequence
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t c0 = 64u * h;    // this half's S columns; its P8 takes the first 16
    bool ok = !dead;
    // this row's Q scale, and the K scales of the sequence; ksc32(j, c) is the scale of
    // keys 32c .. 32c + 31 of KV tile j (its 64-token block, or its own 32-token block)
    const float sq = a.fine
        ? a.q_scale[static_cast<int64_t>(hq) * seq.t_pad + off + qt * kBlkQ + row]
        : a.q_scale[static_cast<int64_t>(hq) * (seq.t_pad / kBlkQ) + off / kBlkQ + qt];
    const int kblk = a.fine ? kBlkKFine : kBlkK;
    const float* ksc = a.k_scale + static_cast<int64_t>(hk) * (seq.t_pad / kblk) + off / kblk;
    auto ksc32 = [&](int j, int c) { return a.fine ? ksc[4 * j + c] : ksc[2 * j + (c >> 1)]; };

    // both S buffers start free
    if (ok && lane == 0) { mbar_arrive(bar_sfree(0)); mbar_arrive(bar_sfree(1)); }

    float m = -INFINITY, l = 0.0f;
    for (int j = 0; j < nkv && ok; ++j) {
      const int buf = j & 1;
      const uint32_t tS = tmem + lane_base + 128u * buf;
      // logit factors of this half's two 32-key chunks
      const float cka = __fmul_rn(__fmul_rn(sq, ksc32(j, 2 * h)), a.scale_log2);
      const float ckb = __fmul_rn(__fmul_rn(sq, ksc32(j, 2 * h + 1)), a.scale_log2);
      const bool masked = (a.causal && j == qt) || (j + 1) * kKvTile > n;
      const int kv0 = j * kKvTile + 64 * h;  // first key of this half
      auto dropped = [&](int key) { return key >= n || (a.causal && key > grow); };
      ok = __all_sync(0xffffffffu, mbar_wait(bar_sfull(buf), (j >> 1) & 1, 0x301 + h));
      if (!ok) break;
      tc_fence_after();

      // pass 1: the largest magic-offset score of this half (masked keys read as 0,
      // below every valid value 12582912 + S)
      uint32_t ra[32], rb[32];
      tmem_ld32(tS + c0, ra);
      tmem_ld32(tS + c0 + 32u, rb);
      tmem_wait_ld_tied(ra, rb);
      uint32_t keep_a = 0xFFFFFFFFu, keep_b = 0xFFFFFFFFu;
      if (masked) {
        keep_a = 0u;
        keep_b = 0u;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          if (dropped(kv0 + i)) ra[i] = 0u; else keep_a |= 1u << i;
          if (dropped(kv0 + 32 + i)) rb[i] = 0u; else keep_b |= 1u << i;
        }
      }
      // this half's max logit (log2 units): each 32-key chunk's largest score times the
      // chunk's factor (the same as the largest score of the half times its factor when
      // both chunks share one K block: rounding is monotone)
      const float hma = max32(ra, 0.0f), hmb = max32(rb, 0.0f);
      const float hs = fmaxf(hma > 1.0e6f ? __fmul_rn(__fsub_rn(hma, kMagic), cka) : -INFINITY,
                             hmb > 1.0e6f ? __fmul_rn(__fsub_rn(hmb, kMagic), ckb) : -INFINITY);
      // exchange with the other softmax warp of this lane quarter
      xchg[(buf * 2 + h) * 128 + row] = hs;
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_xchg(buf, quarter));
      ok = __all_sync(0xffffffffu, mbar_wait(bar_xchg(buf, quarter), (j >> 1) & 1, 0x305 + h));
      if (!ok) break;
      const float mt = fmaxf(hs, xchg[(buf * 2 + (1 - h)) * 128 + row]);
      const float m_new = fmaxf(m, mt);
      const float alpha = ex2(m - m_new);
      const float nbias = __fsub_rn(kLog2_448, m_new);
      if (h == 0) alph[buf * 128 + row] = alpha;

      // pass 2 on the same registers: p = 448 * 2^(u - m'), e4m3 P8 into this half's
      // first 16 columns
      f2 acc = make_float2(0.0f, 0.0f);
      uint32_t w[8];
      if (masked) p8_chunk<true>(ra, cka, nbias, acc, w, keep_a);
      else p8_chunk<false>(ra, cka, nbias, acc, w, 0u);
      tmem_st8(tS + c0, w);
      if (masked) p8_chunk<true>(rb, ckb, nbias, acc, w, keep_b);
      else p8_chunk<false>(rb, ckb, nbias, acc, w, 0u);
      tmem_st8(tS + c0 + 8u, w);
      l = l * alpha + (f2_lo(acc) + f2_hi(acc));
      m = m_new;
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) { mbar_arrive(bar_pfull(buf)); mbar_arrive(bar_sfree(buf)); }
    }
    // hand the row's partial sum (and, from the first half, its max) to the epilogue
    lfin[h * 128 + row] = l;
    if (h == 0) lfin[256 + row] = m;
    __syncwarp();
    if (lane == 0) mbar_arrive(bar_epi);
  } else {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kCorrectionRegs));
    // ============================================================ two-level accumulation
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int grow = qt * kBlkQ + row;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tPV = tmem + lane_base + kColPV;
    const uint32_t tO = tmem + lane_base + kColO;
    bool ok = !dead;

    // both S buffers start free
    if (ok && lane == 0) { mbar_arrive(bar_sfree(0)); mbar_arrive(bar_sfree(1)); }

    for (int j = 0; j < nkv && ok; ++j) {
      const int buf = j & 1;
      ok = __all_sync(0xffffffffu, mbar_wait<true>(bar_pfull(buf), (j >> 1) & 1, 0x401)) &&
           __all_sync(0xffffffffu, mbar_wait<true>(bar_pvfull, j & 1, 0x402));
      if (!ok) break;
      tc_fence_after();
      // PV(j) has read P8(j): buffer j % 2 may take S(j + 2)
      if (lane == 0) mbar_arrive(bar_sfree(buf));
      const f2 al = make_float2(alph[buf * 128 + row], alph[buf * 128 + row]);
      // O = alpha * O + PV_blk, 32 columns at a time (the first tile just copies PV_blk)
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t rp[32], ro[32];
        tmem_ld32(tPV + 32u * c, rp);
        if (j > 0) {
          tmem_ld32(tO + 32u * c, ro);
          tmem_wait_ld_tied(rp, ro);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const f2 o = f2_fma(pair_of(ro, i), al, pair_of(rp, i));
            ro[2 * i] = __float_as_uint(o.x);
            ro[2 * i + 1] = __float_as_uint(o.y);
          }
          tmem_st32(tO + 32u * c, ro);
        } else {
          tmem_wait_ld_tied(rp);
          tmem_st32(tO + 32u * c, rp);
        }
      }
      // PV_blk has been read and O written back: the next PV may overwrite PV_blk
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_pvfree);
    }

    // ---------------------------------------------------------------- epilogue
    ok = ok && __all_sync(0xffffffffu, mbar_wait(bar_epi, 0, 0x403));
    if (ok) {
      tc_fence_after();
      const float l = lfin[row] + lfin[128 + row];
      const float m = lfin[256 + row];
      const float inv_l = 1.0f / l;
      const float* vs = a.v_scale + (static_cast<int64_t>(b) * a.hkv + hk) * D;
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
          for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(ro[i]) * vs[32 * c + i] * inv_l;
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
            m * 0.6931471805599453f + (logf(l) - kLn448);
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
