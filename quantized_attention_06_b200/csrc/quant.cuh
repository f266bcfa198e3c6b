// quant.cuh - smoothing and quantization kernels (HBM-streaming, 16-byte vector loads).
//
// K smoothing and per-block INT8 quantization of Q and K follow the glossary
// page "SageAttention(セージアテンション)" (概要, 主な特徴・仕組み) and the vibecrowd
// repo page "thu-ml--sageattention" (How it works: INT8 QK^T, FP8 PV).
//
// Arithmetic is written with explicit IEEE round-to-nearest intrinsics
// (__fsub_rn, __fmul_rn, __fdiv_rn, __float2int_rn, __ddiv_rn) so that no
// contraction or approximate division can change a code.
//
// Kernels (one 256-thread CTA per block of tokens of one head):
//   k_colsum   fp64 per-channel sums of K over each 128-token padded block
//   k_mean     per (sequence, kv head): mu = fp32(sum / n)
//   v_colmax   per-channel max |V| over each 128-token padded block
//   v_finalize per (sequence, kv head): vmax, v_scale = vmax / 448
//   quant_qk   Q blocks of 128 tokens and smoothed K blocks of 64 tokens -> int8 + scale
//   quant_v    V -> e4m3 with per-channel scale, written token-contiguous (transposed)
//   transpose_v16  V kept in its 16-bit input type, written token-contiguous (the
//              16-bit PV option), and fill_ones for its unit V scales
#pragma once

#include "sage_device.cuh"
#include "seq_table.cuh"

namespace sage {

constexpr int kQuantThreads = 256;

__device__ __forceinline__ uint4 ld_stream16(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// ------------------------------------------------------------------------- K stats
template <typename T, int D, class Seq>
__global__ void __launch_bounds__(kQuantThreads)
k_colsum_kernel(const __grid_constant__ Seq seq, const T* __restrict__ k, int64_t sb, int64_t sh,
                int64_t st, double* __restrict__ partial) {
  constexpr int VPR = D / 8;               // 16-byte vectors per token row
  constexpr int RG = kQuantThreads / VPR;  // rows handled in parallel
  constexpr int IT = kPad / RG;
  __shared__ double red[RG][D];
  const int pb = blockIdx.x, h = blockIdx.y;
  const SeqPos sp = locate(seq, pb * kPad, sb, st);
  const int t0 = pb * kPad - sp.off;
  const int vc = threadIdx.x % VPR, rg = threadIdx.x / VPR;
  const T* src = k + sp.base + h * sh + vc * 8;
  uint4 v[IT];
#pragma unroll
  for (int it = 0; it < IT; ++it) {
    const int t = t0 + rg + it * RG;
    v[it] = (t < sp.n) ? ld_stream16(src + t * st) : make_uint4(0, 0, 0, 0);
  }
  double acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.0;
#pragma unroll
  for (int it = 0; it < IT; ++it) {
    float f[8];
    unpack8<T>(v[it], f);
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] += static_cast<double>(f[i]);
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) red[rg][vc * 8 + i] = acc[i];
  __syncthreads();
  for (int c = threadIdx.x; c < D; c += kQuantThreads) {
    double s = 0.0;
#pragma unroll 4
    for (int g = 0; g < RG; ++g) s += red[g][c];
    partial[(static_cast<int64_t>(h) * (seq.t_pad / kPad) + pb) * D + c] = s;
  }
}

template <int D, class Seq>
__global__ void __launch_bounds__(D)
k_mean_kernel(const __grid_constant__ Seq seq, const double* __restrict__ partial, int hkv,
              float* __restrict__ k_mean) {
  const int b = blockIdx.x, h = blockIdx.y, c = threadIdx.x;
  const int n = seq_len(seq, b);
  const int blk0 = seq_off(seq, b) / kPad;
  const int nblk = (n + kPad - 1) / kPad;
  const double* p = partial + (static_cast<int64_t>(h) * (seq.t_pad / kPad) + blk0) * D + c;
  double s = 0.0;
  for (int i = 0; i < nblk; ++i) s += p[static_cast<int64_t>(i) * D];
  const float mu = (n > 0) ? __double2float_rn(__ddiv_rn(s, static_cast<double>(n))) : 0.0f;
  k_mean[(static_cast<int64_t>(b) * hkv + h) * D + c] = mu;
}

// ------------------------------------------------------------------------- V stats
template <typename T, int D, class Seq>
__global__ void __launch_bounds__(kQuantThreads)
v_colmax_kernel(const __grid_constant__ Seq seq, const T* __restrict__ v, int64_t sb, int64_t sh,
                int64_t st, float* __restrict__ partial) {
  constexpr int VPR = D / 8;
  constexpr int RG = kQuantThreads / VPR;
  constexpr int IT = kPad / RG;
  __shared__ float red[RG][D];
  const int pb = blockIdx.x, h = blockIdx.y;
  const SeqPos sp = locate(seq, pb * kPad, sb, st);
  const int t0 = pb * kPad - sp.off;
  const int vc = threadIdx.x % VPR, rg = threadIdx.x / VPR;
  const T* src = v + sp.base + h * sh + vc * 8;
  uint4 x[IT];
#pragma unroll
  for (int it = 0; it < IT; ++it) {
    const int t = t0 + rg + it * RG;
    x[it] = (t < sp.n) ? ld_stream16(src + t * st) : make_uint4(0, 0, 0, 0);
  }
  float mx[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) mx[i] = 0.0f;
#pragma unroll
  for (int it = 0; it < IT; ++it) {
    float f[8];
    unpack8<T>(x[it], f);
#pragma unroll
    for (int i = 0; i < 8; ++i) mx[i] = fmaxf(mx[i], fabsf(f[i]));
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) red[rg][vc * 8 + i] = mx[i];
  __syncthreads();
  for (int c = threadIdx.x; c < D; c += kQuantThreads) {
    float m = 0.0f;
    for (int g = 0; g < RG; ++g) m = fmaxf(m, red[g][c]);
    partial[(static_cast<int64_t>(h) * (seq.t_pad / kPad) + pb) * D + c] = m;
  }
}

template <int D, class Seq>
__global__ void __launch_bounds__(D)
v_finalize_kernel(const __grid_constant__ Seq seq, const float* __restrict__ partial, int hkv,
                  float* __restrict__ vmax_out, float* __restrict__ v_scale) {
  const int b = blockIdx.x, h = blockIdx.y, c = threadIdx.x;
  const int n = seq_len(seq, b);
  const int blk0 = seq_off(seq, b) / kPad;
  const int nblk = (n + kPad - 1) / kPad;
  const float* p = partial + (static_cast<int64_t>(h) * (seq.t_pad / kPad) + blk0) * D + c;
  float m = 0.0f;
  for (int i = 0; i < nblk; ++i) m = fmaxf(m, p[static_cast<int64_t>(i) * D]);
  const int64_t o = (static_cast<int64_t>(b) * hkv + h) * D + c;
  vmax_out[o] = m;
  v_scale[o] = (m > 0.0f) ? __fdiv_rn(m, 448.0f) : 0.0f;
}

// ------------------------------------------------------------------------- Q/K INT8
struct QKQuantArgs {
  const void* q;
  const void* k;
  int64_t qsb, qsh, qst, ksb, ksh, kst;
  int8_t* q8;
  float* q_scale;
  int8_t* k8;
  float* k_scale;
  const float* k_mean;
  int hq, hkv;
  int nq_blocks;  // hq * t_pad / 128 (the first CTAs); the rest are K blocks
  int fine;       // per-thread granularity: a scale per Q token and per 32-token K block
};

__device__ __forceinline__ float block_max_256(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int w = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) red[w] = v;
  __syncthreads();
  float m = red[0];
#pragma unroll
  for (int i = 1; i < kQuantThreads / 32; ++i) m = fmaxf(m, red[i]);
  return m;
}

__device__ __forceinline__ uint32_t pack_i8x4(int a, int b, int c, int d) {
  return (static_cast<uint32_t>(a) & 0xFFu) | ((static_cast<uint32_t>(b) & 0xFFu) << 8) |
         ((static_cast<uint32_t>(c) & 0xFFu) << 16) | ((static_cast<uint32_t>(d) & 0xFFu) << 24);
}

__device__ __forceinline__ int quant_i8(float x, float r) {
  const int q = __float2int_rn(__fmul_rn(x, r));
  return max(-127, min(127, q));
}

template <typename T, int D, class Seq>
__global__ void __launch_bounds__(kQuantThreads)
quant_qk_kernel(const __grid_constant__ Seq seq, const __grid_constant__ QKQuantArgs a) {
  constexpr int VPR = D / 8;
  constexpr int RG = kQuantThreads / VPR;
  constexpr int ITQ = kBlkQ / RG;  // 8 (d=128) or 4 (d=64)
  static_assert(RG == 16 || RG == 32, "a row group must not straddle a 32-row K block");
  __shared__ float red[kQuantThreads / 32];
  const bool isq = static_cast<int>(blockIdx.x) < a.nq_blocks;
  const int rows = isq ? kBlkQ : kBlkK;
  const int per_head = seq.t_pad / rows;
  const int local = isq ? blockIdx.x : blockIdx.x - a.nq_blocks;
  const int h = local / per_head, pb = local % per_head;
  const int tp = pb * rows;
  const int64_t sb = isq ? a.qsb : a.ksb, sh = isq ? a.qsh : a.ksh, st = isq ? a.qst : a.kst;
  const SeqPos sp = locate(seq, tp, sb, st);
  const int t0 = tp - sp.off;
  const int vc = threadIdx.x % VPR, rg = threadIdx.x / VPR;
  const T* src = reinterpret_cast<const T*>(isq ? a.q : a.k) + sp.base + h * sh + vc * 8;

  float mu[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) mu[i] = 0.0f;
  if (!isq) {
    const float* m = a.k_mean + (static_cast<int64_t>(sp.b) * a.hkv + h) * D + vc * 8;
#pragma unroll
    for (int i = 0; i < 8; ++i) mu[i] = m[i];
  }
  const int iters = rows / RG;
  float x[ITQ][8];
  float amax = 0.0f;
#pragma unroll
  for (int it = 0; it < ITQ; ++it) {
    const int t = t0 + rg + it * RG;
    const bool valid = it < iters && t < sp.n;
    uint4 v = valid ? ld_stream16(src + t * st) : make_uint4(0, 0, 0, 0);
    float f[8];
    unpack8<T>(v, f);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      x[it][i] = valid ? (isq ? f[i] : __fsub_rn(f[i], mu[i])) : 0.0f;
      amax = fmaxf(amax, fabsf(x[it][i]));
    }
  }
  // the scale of each row: one per CTA block, or (fine) one per Q row / 32-row K block
  float rit[ITQ];
  int8_t* dst = (isq ? a.q8 : a.k8) + (static_cast<int64_t>(h) * seq.t_pad + tp) * D + vc * 8;
  if (!a.fine) {
    amax = block_max_256(amax, red);
    const float s = (amax > 0.0f) ? __fdiv_rn(amax, 127.0f) : 0.0f;
    const float r = (amax > 0.0f) ? __fdiv_rn(127.0f, amax) : 0.0f;
#pragma unroll
    for (int it = 0; it < ITQ; ++it) rit[it] = r;
    if (threadIdx.x == 0) (isq ? a.q_scale : a.k_scale)[static_cast<int64_t>(h) * per_head + pb] = s;
  } else if (isq) {
    // the VPR consecutive lanes holding one row reduce its max by shuffles
#pragma unroll
    for (int it = 0; it < ITQ; ++it) {
      float m = 0.0f;
#pragma unroll
      for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(x[it][i]));
#pragma unroll
      for (int o = VPR / 2; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      rit[it] = (m > 0.0f) ? __fdiv_rn(127.0f, m) : 0.0f;
      if (vc == 0 && it < iters)
        a.q_scale[static_cast<int64_t>(h) * seq.t_pad + tp + rg + it * RG] =
            (m > 0.0f) ? __fdiv_rn(m, 127.0f) : 0.0f;
    }
  } else {
    // two 32-row K blocks per CTA: row rg + it * RG (rg < RG) lies in block it * RG / 32
    __shared__ float red2[2][kQuantThreads / 32];
    float m2[2] = {0.0f, 0.0f};
#pragma unroll
    for (int it = 0; it < ITQ; ++it) {
      if (it < iters) {
        const int sb = (it * RG) / kBlkKFine;  // rows it*RG .. it*RG + RG-1, RG in {16, 32}
#pragma unroll
        for (int i = 0; i < 8; ++i) m2[sb] = fmaxf(m2[sb], fabsf(x[it][i]));
      }
    }
#pragma unroll
    for (int b2 = 0; b2 < 2; ++b2) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m2[b2] = fmaxf(m2[b2], __shfl_xor_sync(0xffffffffu, m2[b2], o));
      if ((threadIdx.x & 31) == 0) red2[b2][threadIdx.x >> 5] = m2[b2];
    }
    __syncthreads();
    float r2[2];
#pragma unroll
    for (int b2 = 0; b2 < 2; ++b2) {
      float m = red2[b2][0];
#pragma unroll
      for (int i = 1; i < kQuantThreads / 32; ++i) m = fmaxf(m, red2[b2][i]);
      r2[b2] = (m > 0.0f) ? __fdiv_rn(127.0f, m) : 0.0f;
      if (threadIdx.x == 0)
        a.k_scale[static_cast<int64_t>(h) * (seq.t_pad / kBlkKFine) + pb * 2 + b2] =
            (m > 0.0f) ? __fdiv_rn(m, 127.0f) : 0.0f;
    }
#pragma unroll
    for (int it = 0; it < ITQ; ++it) rit[it] = r2[((it * RG) / kBlkKFine) & 1];
  }
#pragma unroll
  for (int it = 0; it < ITQ; ++it) {
    if (it < iters) {
      const int rr = rg + it * RG;
      const float r = rit[it];
      uint2 o;
      o.x = pack_i8x4(quant_i8(x[it][0], r), quant_i8(x[it][1], r), quant_i8(x[it][2], r),
                      quant_i8(x[it][3], r));
      o.y = pack_i8x4(quant_i8(x[it][4], r), quant_i8(x[it][5], r), quant_i8(x[it][6], r),
                      quant_i8(x[it][7], r));
      *reinterpret_cast<uint2*>(dst + static_cast<int64_t>(rr) * D) = o;
    }
  }
}

// ------------------------------------------------------------------------- V e4m3
struct VQuantArgs {
  const void* v;
  int64_t sb, sh, st;
  const float* vmax;  // [B][Hkv][D]
  uint8_t* v8;        // [Hkv][D][T_pad]
  int hkv;
};

template <typename T, int D, class Seq>
__global__ void __launch_bounds__(kQuantThreads)
quant_v_kernel(const __grid_constant__ Seq seq, const __grid_constant__ VQuantArgs a) {
  // One CTA: one 128-token block of one KV head.  Thread (cg, tg) converts channels
  // 8cg .. 8cg+7 of tokens TPT*tg .. TPT*tg+TPT-1, pairing two tokens of one channel
  // per e4m3x2 conversion, so each channel's TPT codes leave the thread as one
  // TPT-byte word.  The words go into a [D][128] byte tile whose 16-byte chunks are
  // XOR-swizzled by (channel % 8), and each channel row then leaves as 16-byte
  // stores of the token-contiguous output.
  constexpr int CG = D / 8;                  // channel groups (16-byte input vectors)
  constexpr int TG = kQuantThreads / CG;     // token groups
  constexpr int TPT = kPad / TG;             // tokens per thread: 8 (d = 128) or 4 (d = 64)
  static_assert(TPT == 4 || TPT == 8, "tile shape");
  __shared__ __align__(16) uint8_t tile[D * kPad];
  const int pb = blockIdx.x, h = blockIdx.y;
  const SeqPos sp = locate(seq, pb * kPad, a.sb, a.st);
  const int t0 = pb * kPad - sp.off;
  const int cg = threadIdx.x % CG, tg = threadIdx.x / CG;
  const T* src = reinterpret_cast<const T*>(a.v) + sp.base + h * a.sh + cg * 8;
  float r[8];
  {
    const float* vm = a.vmax + (static_cast<int64_t>(sp.b) * a.hkv + h) * D + cg * 8;
#pragma unroll
    for (int i = 0; i < 8; ++i) r[i] = (vm[i] > 0.0f) ? __fdiv_rn(448.0f, vm[i]) : 0.0f;
  }
  // codes[c][u]: e4m3 of channel 8cg+c for tokens (2u, 2u+1) of this thread, 16 bits
  uint32_t codes[8][TPT / 2];
#pragma unroll
  for (int u = 0; u < TPT / 2; ++u) {
    const int ta = t0 + TPT * tg + 2 * u, tb = ta + 1;
    const bool va = ta < sp.n, vb = tb < sp.n;
    float fa[8], fb[8];
    unpack8<T>(va ? ld_stream16(src + static_cast<int64_t>(ta) * a.st) : make_uint4(0, 0, 0, 0), fa);
    unpack8<T>(vb ? ld_stream16(src + static_cast<int64_t>(tb) * a.st) : make_uint4(0, 0, 0, 0), fb);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const uint32_t two = e4m3x2(__fmul_rn(fa[c], r[c]), __fmul_rn(fb[c], r[c]));
      codes[c][u] = two & ((va ? 0xFFu : 0u) | (vb ? 0xFF00u : 0u));  // padding tokens: 0
    }
  }
  // channel order rotated by cg: lanes cg and cg + 8 share a bank, no more
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int c = (k + cg) & 7;
    const int ch = cg * 8 + c;
    const int tok = TPT * tg;  // first token of this thread within the block
    const int off = ch * kPad + ((((tok >> 4) ^ ch) & 7) << 4) + (tok & 15);
    uint32_t w0 = 0u, w1 = 0u;
#pragma unroll
    for (int u = 0; u < TPT / 2; ++u) {
      // select this channel's codes without a dynamically indexed register array
      uint32_t v = 0u;
#pragma unroll
      for (int cc = 0; cc < 8; ++cc) v = (cc == c) ? codes[cc][u] : v;
      if (u < 2) w0 |= v << (16 * u);
      else w1 |= v << (16 * (u - 2));
    }
    if (TPT == 8) *reinterpret_cast<uint2*>(tile + off) = make_uint2(w0, w1);
    else *reinterpret_cast<uint32_t*>(tile + off) = w0;
  }
  __syncthreads();
  // each channel row of the tile is 128 contiguous output bytes: 8 threads x 16 B
  uint8_t* dst = a.v8 + static_cast<int64_t>(h) * D * seq.t_pad + pb * kPad;
  for (int i = threadIdx.x; i < D * 8; i += kQuantThreads) {
    const int ch = i >> 3, j = i & 7;
    const uint4 w = *reinterpret_cast<const uint4*>(tile + ch * kPad + ((j ^ (ch & 7)) << 4));
    *reinterpret_cast<uint4*>(dst + static_cast<int64_t>(ch) * seq.t_pad + j * 16) = w;
  }
}

// ------------------------------------------------------------------------- V 16-bit
// The 16-bit PV option keeps V at its input values: the same token-contiguous
// [Hkv][D][T_pad] layout as the e4m3 codes, two bytes per entry.  One CTA: one
// 128-token block of one KV head; thread (cg, tg) holds channels 8cg .. 8cg+7 of
// tokens TPT*tg .. TPT*tg+TPT-1 and writes each channel's TPT values as one word into
// a [D][128] tile whose 16-byte chunks are XOR-swizzled by channel; the rows then
// leave as 16-byte stores.
template <typename T, int D, class Seq>
__global__ void __launch_bounds__(kQuantThreads)
transpose_v16_kernel(const __grid_constant__ Seq seq, const __grid_constant__ VQuantArgs a) {
  constexpr int CG = D / 8;
  constexpr int TG = kQuantThreads / CG;
  constexpr int TPT = kPad / TG;  // 8 (d = 128) or 4 (d = 64)
  static_assert(TPT == 4 || TPT == 8, "tile shape");
  __shared__ __align__(16) uint8_t tile[D * kPad * 2];  // D rows of 256 bytes
  const int pb = blockIdx.x, h = blockIdx.y;
  const SeqPos sp = locate(seq, pb * kPad, a.sb, a.st);
  const int t0 = pb * kPad - sp.off;
  const int cg = threadIdx.x % CG, tg = threadIdx.x / CG;
  const T* src = reinterpret_cast<const T*>(a.v) + sp.base + h * a.sh + cg * 8;
  uint32_t raw[TPT][4];  // token u: channels 8cg .. 8cg+7 as 8 x 16 bits
#pragma unroll
  for (int u = 0; u < TPT; ++u) {
    const int t = t0 + TPT * tg + u;
    const uint4 x = (t < sp.n) ? ld_stream16(src + static_cast<int64_t>(t) * a.st) : make_uint4(0, 0, 0, 0);
    raw[u][0] = x.x; raw[u][1] = x.y; raw[u][2] = x.z; raw[u][3] = x.w;
  }
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int c = (k + cg) & 7;  // rotated by cg: fewer threads of a warp on one bank
    const int ch = cg * 8 + c;
    const int tok = TPT * tg;
    uint32_t w[TPT / 2];
#pragma unroll
    for (int u = 0; u < TPT; u += 2) {
      uint32_t lo = 0u, hi = 0u;
#pragma unroll
      for (int cc = 0; cc < 8; ++cc) {  // no dynamically indexed register array
        if (cc == c) {
          lo = (raw[u][cc >> 1] >> (16 * (cc & 1))) & 0xFFFFu;
          hi = (raw[u + 1][cc >> 1] >> (16 * (cc & 1))) & 0xFFFFu;
        }
      }
      w[u / 2] = lo | (hi << 16);
    }
    const int off = ch * (kPad * 2) + ((((tok >> 3) ^ ch) & 15) << 4) + (tok & 7) * 2;
    if constexpr (TPT == 8) *reinterpret_cast<uint4*>(tile + off) = make_uint4(w[0], w[1], w[2], w[3]);
    else *reinterpret_cast<uint2*>(tile + off) = make_uint2(w[0], w[1]);
  }
  __syncthreads();
  uint8_t* dst = reinterpret_cast<uint8_t*>(a.v8) + (static_cast<int64_t>(h) * D * seq.t_pad + pb * kPad) * 2;
  for (int i = threadIdx.x; i < D * 16; i += kQuantThreads) {
    const int ch = i >> 4, j = i & 15;
    const uint4 w = *reinterpret_cast<const uint4*>(tile + ch * (kPad * 2) + (((j ^ ch) & 15) << 4));
    *reinterpret_cast<uint4*>(dst + static_cast<int64_t>(ch) * seq.t_pad * 2 + j * 16) = w;
  }
}

__global__ void fill_ones_kernel(float* __restrict__ x, int64_t n) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < n) x[i] = 1.0f;
}

}  // namespace sage
