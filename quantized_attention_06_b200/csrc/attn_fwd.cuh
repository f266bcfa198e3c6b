// attn_fwd.cuh - quantized attention forward on sm_100a tensor cores.
//
// Method (SageAttention): vibecrowd repo page "thu-ml--sageattention", How it
// works (INT8 QK^T, FP8 PV, two-level accumulation for PV); heatdrop review
// "2–5× attention speedups without the accuracy apology tour", The interesting
// bit (two-level accumulation inside FP8 tensor cores) and Key highlights (GQA,
// variable lengths); glossary page "SageAttention(セージアテンション)" (FlashAttention-
// compatible online softmax).
//
// CTA = one (sequence, query head, pair of 128-row Q tiles).  12 warps in three
// warpgroups; the producer warpgroup gives registers to the softmax warpgroups
// (setmaxnreg: 128 x 40 + 256 x 232 = 384 x 168, the launch allocation):
//   warp 0      TMA producer: both Q tiles once, then K / V tiles into 3-stage rings
//   warp 1      TMEM owner and MMA issuer (one thread):
//                 S_t  = Q8_t K8^T      tcgen05.mma kind::i8     -> TMEM s32 [128 x 128]
//                 PV_t = P8_t V8       tcgen05.mma kind::f8f6f4 (A = P8 in TMEM) -> TMEM f32 [128 x d]
//   warps 2-3   idle
//   warps 4-7   softmax + correction for Q tile 0 (one thread per query row)
//   warps 8-11  softmax + correction for Q tile 1
// TMEM columns: [0,128) S/P of tile 0, [128,256) S/P of tile 1,
//               [256,256+d) PV of tile 0, [384,384+d) PV of tile 1.
// P8 of tile t is written over the first 32 columns of its S region (4 e4m3 per
// column); the MMA that overwrites them with the next S is issued after the PV
// MMA that reads them, and tcgen05.mma ops of one thread execute in issue order.
//
// Per KV tile j the softmax thread of query row i (log2 domain, u = x * log2 e):
//   u_j   = S_ij * (q_scale * k_scale_j * sm_scale * log2 e)   (S read as 12582912 + S)
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

constexpr int kAttnThreads = 384;
constexpr int kAttnLaunchRegs = 168;  // 65536 / 384 rounded down to a multiple of 8
constexpr int kProducerRegs = 40;
constexpr int kSoftmaxRegs = 232;
static_assert(128 * kProducerRegs + 256 * kSoftmaxRegs <= kAttnThreads * kAttnLaunchRegs,
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
};

template <int D>
struct AttnSmem {
  static constexpr int kTileQ = kBlkQ * D;      // bytes of one Q (or K) tile
  static constexpr int kTileV = D * kKvTile;    // bytes of one V^T tile
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQOff + 2 * kTileQ;
  static constexpr int kVOff = kKOff + kKStages * kTileQ;
  static constexpr int kBarOff = kVOff + kVStages * kTileV;
  // barriers: q_full, k_full[3], k_empty[3], v_full[3], v_empty[3], s_full[2], p_full[2],
  // pv_full[2], mma_done, s_free[2]  -> 22 x 8 bytes, then the TMEM address slot
  static constexpr int kNumBars = 22;
  static constexpr int kSlotOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kSlotOff + 16;
  static constexpr int kAlloc = kBytes + 1024;  // room to align the base to 1024
};

__device__ __forceinline__ float i2f_exact(uint32_t s) {
  // exact int32 -> fp32 for |s| < 2^22: place s in the mantissa of 1.5 * 2^23
  return __fsub_rn(__int_as_float(static_cast<int>(s) + 0x4B400000), 12582912.0f);
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^t in plain IEEE fp32 operations, so that the P8 code it decides can be
// reproduced exactly on any host: Cody-Waite split t = n + f with n = rint(t)
// taken by magic-number rounding (r = t + 1.5 * 2^23, bits(r) = 0x4B400000 + n)
// and f = t - (r - 1.5 * 2^23) in [-1/2, 1/2], a degree-3 polynomial for 2^f
// (coefficients fitted for minimal relative error with the constant term fixed at
// 1; max relative error 1.0e-4), and n added to the exponent field, clamped below
// at -125 so the result stays a normal number.
constexpr float kExp2C1 = 0.693282962f;   // 0x3f317afe
constexpr float kExp2C2 = 0.242211089f;   // 0x3e78062f
constexpr float kExp2C3 = 0.0550086424f;  // 0x3d6150be
constexpr int kExpClampBits = 0x4B400000 - 125;
__device__ __forceinline__ float exp2_poly(float t) {
  const float r = __fadd_rn(t, 12582912.0f);
  const float f = __fsub_rn(t, __fsub_rn(r, 12582912.0f));
  float p = __fmaf_rn(kExp2C3, f, kExp2C2);
  p = __fmaf_rn(p, f, kExp2C1);
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

// 32 lanes x 32 consecutive columns of TMEM all set to kMagicBits.
__device__ __forceinline__ void tmem_fill_magic32(uint32_t taddr) {
  const uint32_t v = kMagicBits;
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,"
      "%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1};" ::"r"(taddr),
      "r"(v)
      : "memory");
}

// max over 32 magic-offset scores (masked entries hold 0, below every valid value)
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
  const f2 C3 = f2_make(kExp2C3, kExp2C3);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    f2 pp[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const f2 t = f2_fma(f2_add(pair_of(r, 2 * i + h), NM), CK, NB);
      const f2 rr = f2_add(t, M);
      const f2 f = f2_fma(f2_add(rr, NM), NEG1, t);
      f2 p = f2_fma(C3, f, C2);
      p = f2_fma(p, f, C1);
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
  constexpr uint32_t kColS0 = 0, kColPV0 = 256;

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
  auto bar_s = [&](int t) { return bar0 + 8u * (13 + t); };
  auto bar_p = [&](int t) { return bar0 + 8u * (15 + t); };
  auto bar_pv = [&](int t) { return bar0 + 8u * (17 + t); };
  const uint32_t bar_done = bar0 + 8u * 19;
  auto bar_sf = [&](int t) { return bar0 + 8u * (20 + t); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kSlotOff);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---------------------------------------------------------------- work item
  int b, hq, pair;
  {
    int idx = blockIdx.x;
    if constexpr (std::is_same<Seq, SeqDense>::value) {
      const int nq = (seq_len(seq, 0) + kBlkQ - 1) / kBlkQ;
      const int pairs = (nq + 1) / 2;
      const int g = idx % a.group; idx /= a.group;
      pair = idx % pairs; idx /= pairs;
      const int hk = idx % a.hkv;
      b = idx / a.hkv;
      hq = hk * a.group + g;
      if (a.causal) pair = pairs - 1 - pair;  // heaviest pairs first
    } else {
      int lo = 0, hi = seq.nseq - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (seq.cta[mid] <= idx) lo = mid; else hi = mid - 1;
      }
      while (lo + 1 < seq.nseq && seq.cta[lo + 1] <= idx) ++lo;
      b = lo;
      idx -= seq.cta[b];
      const int nq = (seq_len(seq, b) + kBlkQ - 1) / kBlkQ;
      const int pairs = (nq + 1) / 2;
      const int g = idx % a.group; idx /= a.group;
      pair = idx % pairs; idx /= pairs;
      hq = idx * a.group + g;
      if (a.causal) pair = pairs - 1 - pair;
    }
  }
  const int hk = hq / a.group;
  const int n = seq_len(seq, b);
  const int off = seq_off(seq, b);
  const int nq_tiles = (n + kBlkQ - 1) / kBlkQ;
  const int nkv_all = (n + kKvTile - 1) / kKvTile;
  int qt[2], nkv[2];
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    qt[t] = 2 * pair + t;
    nkv[t] = (qt[t] < nq_tiles) ? (a.causal ? qt[t] + 1 : nkv_all) : 0;
  }
  const int n_iter = max(nkv[0], nkv[1]);

  // ---------------------------------------------------------------- set-up
  if (threadIdx.x == 0) {
    mbar_init(bar_q(), 1);
    for (int s = 0; s < kKStages; ++s) { mbar_init(bar_kf(s), 1); mbar_init(bar_ke(s), 1); }
    for (int s = 0; s < kVStages; ++s) { mbar_init(bar_vf(s), 1); mbar_init(bar_ve(s), 1); }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar_s(t), 1);
      mbar_init(bar_p(t), 4);  // one arrival per softmax warp
      mbar_init(bar_pv(t), 1);
      mbar_init(bar_sf(t), 4);  // one arrival per softmax warp: S region re-armed
    }
    mbar_init(bar_done, 1);
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
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const bool dead = watchdog_tripped();

  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kProducerRegs));
   if (warp == 0) {
    // ============================================================ TMA producer
    if (lane == 0 && !dead) {
      bool ok = true;
      const int qbytes = (nkv[1] > 0 ? 2 : 1) * L::kTileQ;
      mbar_arrive_expect_tx(bar_q(), qbytes);
      for (int t = 0; t < 2; ++t)
        if (nkv[t] > 0)
          tma_load_2d(sbase + L::kQOff + t * L::kTileQ, &tmap_q, 0,
                      hq * seq.t_pad + off + qt[t] * kBlkQ, bar_q());
      int nk = 0, nv = 0;  // loads issued
      for (int j = 0; j < n_iter && ok; ++j) {
        const int ks = j % kKStages, vs = j % kVStages;
        if (j >= kKStages) ok = mbar_wait(bar_ke(ks), ((j / kKStages) - 1) & 1, 0x101);
        if (!ok) break;
        mbar_arrive_expect_tx(bar_kf(ks), L::kTileQ);
        tma_load_2d(sbase + L::kKOff + ks * L::kTileQ, &tmap_k, 0,
                    hk * seq.t_pad + off + j * kKvTile, bar_kf(ks));
        ++nk;
        if (j >= kVStages) ok = mbar_wait(bar_ve(vs), ((j / kVStages) - 1) & 1, 0x102);
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
    }
  } else if (warp == 1) {
    // ============================================================ MMA issuer
    if (lane == 0 && !dead) {
      // descriptors differ only in their start-address field (bits 0-13, address >> 4):
      // keep one base per operand and add offsets at issue time
      const uint64_t dq = sdesc_kmajor(sbase + L::kQOff, kSboQK, kSwizzle);
      const uint64_t dk = sdesc_kmajor(sbase + L::kKOff, kSboQK, kSwizzle);
      const uint64_t dv = sdesc_kmajor(sbase + L::kVOff, 1024u, 2u);
      auto issue_s = [&](int t, int ks) {
        const uint64_t aq = dq + static_cast<uint64_t>((t * L::kTileQ) >> 4);
        const uint64_t bk = dk + static_cast<uint64_t>((ks * L::kTileQ) >> 4);
        const uint32_t d_tmem = tmem + kColS0 + 128u * t;
#pragma unroll
        for (int s = 0; s < D / 32; ++s)
          mma_i8_ss(d_tmem, aq + 2u * s, bk + 2u * s, kIdescS, 1u);
        tc_commit(bar_s(t));
      };
      auto issue_pv = [&](int t, int vs) {
        const uint64_t bv = dv + static_cast<uint64_t>((vs * L::kTileV) >> 4);
        const uint32_t d_tmem = tmem + kColPV0 + 128u * t;
        const uint32_t a_tmem = tmem + kColS0 + 128u * t;
#pragma unroll
        for (int s = 0; s < kKvTile / 32; ++s)
          mma_f8_ts(d_tmem, a_tmem + 8u * s, bv + 2u * s, kIdescPV, s > 0 ? 1u : 0u);
        tc_commit(bar_pv(t));
      };
      // S_t(j) accumulates onto the magic bit pattern the softmax warps wrote into the
      // S region (re-armed after PV_t(j-1) consumed P_t(j-1)): wait for that first
      bool ok = mbar_wait(bar_q(), 0, 0x201) && mbar_wait(bar_kf(0), 0, 0x202);
      for (int t = 0; t < 2 && ok; ++t) {
        if (nkv[t] == 0) continue;
        ok = mbar_wait(bar_sf(t), 0, 0x207 + t);
        if (!ok) break;
        tc_fence_after();
        issue_s(t, 0);
      }
      if (ok) tc_commit(bar_ke(0));
      for (int j = 0; j < n_iter && ok; ++j) {
        const int vs = j % kVStages;
        bool v_ready = false, k_ready = false;
        const int jn = j + 1, ksn = jn % kKStages;
        bool issued_next = false;
        for (int t = 0; t < 2 && ok; ++t) {
          if (j >= nkv[t]) continue;
          ok = mbar_wait(bar_p(t), j & 1, 0x203 + t);
          if (ok && !v_ready) { ok = mbar_wait(bar_vf(vs), (j / kVStages) & 1, 0x205); v_ready = true; }
          if (!ok) break;
          tc_fence_after();
          issue_pv(t, vs);
          if (jn < nkv[t]) {
            if (!k_ready) { ok = mbar_wait(bar_kf(ksn), (jn / kKStages) & 1, 0x206); k_ready = true; }
            if (ok) ok = mbar_wait(bar_sf(t), jn & 1, 0x207 + t);
            if (!ok) break;
            tc_fence_after();
            issue_s(t, ksn);
            issued_next = true;
          }
        }
        if (!ok) break;
        if (issued_next) tc_commit(bar_ke(ksn));
        tc_commit(bar_ve(vs));
      }
      // every MMA issued by this thread has completed before TMEM is released
      tc_commit(bar_done);
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait_sleep(bar_done, 0) && global_timer_ns() - t0 < kWaitLimitNs) {}
    }
   }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs));
    // ============================================================ softmax + correction
    const int t = (warp - 4) >> 2;  // Q tile of this warpgroup
    const int quarter = warp & 3;   // TMEM lane quarter this warp may access
    const int row = quarter * 32 + lane;
    const int grow = qt[t] * kBlkQ + row;  // query index within the sequence
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_base + kColS0 + 128u * t;
    const uint32_t tPV = tmem + lane_base + kColPV0 + 128u * t;

    f2 o2[D / 2];  // running output, columns (2c, 2c+1) in pair c
#pragma unroll
    for (int c = 0; c < D / 2; ++c) o2[c] = make_float2(0.0f, 0.0f);
    float m = -INFINITY, l = 0.0f;
    bool ok = !dead;
    const float sq = (nkv[t] > 0) ? a.q_scale[static_cast<int64_t>(hq) * (seq.t_pad / kBlkQ) +
                                              off / kBlkQ + qt[t]]
                                  : 0.0f;
    const float* ksc = a.k_scale + static_cast<int64_t>(hk) * (seq.t_pad / kBlkK) + off / kBlkK;

    // arm the S region: the first QK^T accumulates onto the magic bit pattern
    if (ok && nkv[t] > 0) {
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_fill_magic32(tS + 32u * c);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_sf(t));
    }

    for (int j = 0; j < nkv[t] && ok; ++j) {
      const float ck0 = __fmul_rn(__fmul_rn(sq, ksc[2 * j]), a.scale_log2);
      const float ck1 = __fmul_rn(__fmul_rn(sq, ksc[2 * j + 1]), a.scale_log2);
      const bool masked = (a.causal && j == qt[t]) || (j + 1) * kKvTile > n;
      const int kv0 = j * kKvTile;
      auto dropped = [&](int key) { return key >= n || (a.causal && key > grow); };
      ok = __all_sync(0xffffffffu, mbar_wait(bar_s(t), j & 1, 0x301 + t));
      if (!ok) break;
      tc_fence_after();

      // pass 1: largest score of each 64-key half (masked keys read as 0 < every valid value)
      float hmax[2];
      {
        uint32_t ra[32], rb[32];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          tmem_ld32(tS + 64u * h, ra);
          tmem_ld32(tS + 64u * h + 32u, rb);
          tmem_wait_ld_tied(ra, rb);
          if (masked) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              if (dropped(kv0 + 64 * h + i)) ra[i] = 0u;
              if (dropped(kv0 + 64 * h + 32 + i)) rb[i] = 0u;
            }
          }
          hmax[h] = max32(rb, max32(ra, 0.0f));
        }
      }
      // an all-masked half leaves 0; valid values are at least 12582912 - 2^21
      const float mt = fmaxf(hmax[0] > 1.0e6f ? __fmul_rn(__fsub_rn(hmax[0], kMagic), ck0) : -INFINITY,
                             hmax[1] > 1.0e6f ? __fmul_rn(__fsub_rn(hmax[1], kMagic), ck1) : -INFINITY);
      const float m_new = fmaxf(m, mt);
      const float alpha = ex2(m - m_new);
      const float nbias = __fsub_rn(kLog2_448, m_new);

      // pass 2: p = 448 * 2^(u - m'), running sum, e4m3 P8 into TMEM columns 0-31,
      // columns 32-127 re-armed with the magic pattern once read
      f2 acc = make_float2(0.0f, 0.0f);
      {
        uint32_t ra[32], rb[32];
        uint32_t w[8];
        auto finish = [&](uint32_t (&r)[32], int c) {
          const float ck = c < 2 ? ck0 : ck1;
          if (masked) {
            uint32_t keep = 0u;
#pragma unroll
            for (int i = 0; i < 32; ++i) keep |= dropped(kv0 + 32 * c + i) ? 0u : (1u << i);
            p8_chunk<true>(r, ck, nbias, acc, w, keep);
          } else {
            p8_chunk<false>(r, ck, nbias, acc, w, 0u);
          }
          tmem_st8(tS + 8u * c, w);
          if (c > 0) tmem_fill_magic32(tS + 32u * c);
        };
        tmem_ld32(tS, ra);
        tmem_wait_ld_tied(ra);
        tmem_ld32(tS + 32u, rb);
        finish(ra, 0);
        tmem_wait_ld_tied(rb);
        tmem_ld32(tS + 64u, ra);
        finish(rb, 1);
        tmem_wait_ld_tied(ra);
        tmem_ld32(tS + 96u, rb);
        finish(ra, 2);
        tmem_wait_ld_tied(rb);
        finish(rb, 3);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_p(t));
      l = l * alpha + (f2_lo(acc) + f2_hi(acc));
      m = m_new;

      // two-level accumulation: O = alpha * O + PV_blk (PV_blk fresh in TMEM for this tile)
      ok = __all_sync(0xffffffffu, mbar_wait(bar_pv(t), j & 1, 0x303 + t));
      if (!ok) break;
      tc_fence_after();
      if (j + 1 < nkv[t]) {  // P consumed: re-arm columns 0-31 for the next QK^T
        tmem_fill_magic32(tS);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_sf(t));
      }
      {
        const f2 al = f2_make(alpha, alpha);
        uint32_t ra[32], rb[32];
        auto accum = [&](const uint32_t (&r)[32], int c) {
#pragma unroll
          for (int i = 0; i < 16; ++i) o2[16 * c + i] = f2_fma(o2[16 * c + i], al, pair_of(r, i));
        };
        tmem_ld32(tPV, ra);
        tmem_wait_ld_tied(ra);
#pragma unroll
        for (int c = 0; c < D / 32; c += 2) {
          tmem_ld32(tPV + 32u * (c + 1), rb);
          accum(ra, c);
          tmem_wait_ld_tied(rb);
          if (c + 2 < D / 32) tmem_ld32(tPV + 32u * (c + 2), ra);
          accum(rb, c + 1);
          if (c + 2 < D / 32) tmem_wait_ld_tied(ra);
        }
      }
    }

    // ---------------------------------------------------------------- epilogue
    if (ok && nkv[t] > 0 && grow < n) {
      const float inv_l = 1.0f / l;
      const float* vs = a.v_scale + (static_cast<int64_t>(b) * a.hkv + hk) * D;
      const int64_t orow = seq_base(seq, b, a.osb, a.ost) + hq * a.osh + static_cast<int64_t>(grow) * a.ost;
      if (a.out_dtype == 2) {
        float* dst = reinterpret_cast<float*>(a.out) + orow;
#pragma unroll
        for (int c = 0; c < D; c += 4) {
          float4 v = make_float4(f2_lo(o2[c / 2]) * vs[c] * inv_l, f2_hi(o2[c / 2]) * vs[c + 1] * inv_l,
                                 f2_lo(o2[c / 2 + 1]) * vs[c + 2] * inv_l, f2_hi(o2[c / 2 + 1]) * vs[c + 3] * inv_l);
          *reinterpret_cast<float4*>(dst + c) = v;
        }
      } else if (a.out_dtype == 1) {
        __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(a.out) + orow;
#pragma unroll
        for (int c = 0; c < D; c += 8) {
          __align__(16) __nv_bfloat16 h8[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) h8[i] = __float2bfloat16_rn(((i & 1) ? f2_hi(o2[(c + i) / 2]) : f2_lo(o2[(c + i) / 2])) * vs[c + i] * inv_l);
          *reinterpret_cast<uint4*>(dst + c) = *reinterpret_cast<const uint4*>(h8);
        }
      } else {
        __half* dst = reinterpret_cast<__half*>(a.out) + orow;
#pragma unroll
        for (int c = 0; c < D; c += 8) {
          __align__(16) __half h8[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) h8[i] = __float2half_rn(((i & 1) ? f2_hi(o2[(c + i) / 2]) : f2_lo(o2[(c + i) / 2])) * vs[c + i] * inv_l);
          *reinterpret_cast<uint4*>(dst + c) = *reinterpret_cast<const uint4*>(h8);
        }
      }
      if (a.lse != nullptr)
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
