// quant_fused.cuh - the whole quantization of Q, K and V in one cooperative launch.
//
// The same arithmetic as the separate kernels in quant.cuh (K smoothing and INT8
// blocks: glossary page "SageAttention(セージアテンション)", 概要 / 主な特徴・仕組み;
// INT8 QK^T and FP8 V: vibecrowd repo page "thu-ml--sageattention", How it works),
// organised for B200: one persistent CTA per SM walks tiles of 128 tokens x d, each
// brought into shared memory by TMA (128-byte swizzled boxes of 64 channels) through
// a 4-stage ring, so the next tiles stream in while the current one is reduced and
// written out.  Three phases, separated by grid-wide barriers (the launch is
// cooperative, so every CTA is resident):
//   1. Q tiles are quantized (their scales need nothing else); K tiles give fp64
//      per-channel sums and V tiles per-channel max |v| (one partial per tile)
//   2. per (sequence, KV head, channel): mu = fp32(sum / n), vmax, v_scale = vmax/448
//   3. K tiles are smoothed and quantized; V tiles are quantized to e4m3 (or, with
//      the 16-bit PV option, only transposed) and written token-contiguous
// Every code, scale and mean is bit-identical to the separate kernels: the same
// IEEE round-to-nearest intrinsics in the same order.
#pragma once

#include <cooperative_groups.h>

#include "quant.cuh"
#include "sage_device.cuh"
#include "seq_table.cuh"

namespace sage {

constexpr int kFusedThreads = 512;
constexpr int kFusedStages = 4;

struct FusedQuantArgs {
  int8_t* q8;
  float* q_scale;
  int8_t* k8;
  float* k_scale;
  float* k_mean;   // [B][Hkv][D]
  void* v8;        // [Hkv][D][T_pad], e4m3 codes or 16-bit values
  float* v_scale;  // [B][Hkv][D]
  double* ksum;    // [Hkv][T_pad/128][D] per-tile partial sums of K
  float* vpart;    // [Hkv][T_pad/128][D] per-tile partial max |V|
  float* vmax;     // [B][Hkv][D]
  int hq, hkv, nblk, batch;
  int fine;  // per-thread granularity: a scale per Q token and per 32-token K block
  int pv16;  // V stays 16-bit (transposed only)
  // positions (1..3) of the token, head and batch dimensions in the 4-D tensor maps
  int dim_tok, dim_head, dim_batch;
};

__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                            int c2, int c3, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(bar)
      : "memory");
}

template <int D>
struct FusedCfg {
  static constexpr int kTile = kPad * D * 2;          // bytes of one 128-token tile
  static constexpr int kBox = kPad * 128;             // bytes of one 64-channel box
  static constexpr int kRedOff = kFusedStages * kTile;
  static constexpr int kRedBytes = 16 * D * 8;        // [warp][channel] fp64 partials
  static constexpr int kBarOff = kRedOff + kRedBytes;
  static constexpr int kBytes = kBarOff + kFusedStages * 8;
  static constexpr int kAlloc = kBytes + 1024;
};

// Byte offset of 16-byte chunk c (8 channels 8c .. 8c+7) of row r in a tile: chunks
// 0-7 sit in the first 64-channel box, 8-15 in the second, each a 128-byte-swizzled
// [128 rows][128 B] image.
template <int D>
__device__ __forceinline__ uint32_t tile_off(int r, int c) {
  return static_cast<uint32_t>((c >> 3) * FusedCfg<D>::kBox + r * 128 + ((((c & 7) ^ r) & 7) << 4));
}

__device__ __forceinline__ uint4 lds16(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

// max over the 512 threads of a CTA (every thread returns the result)
__device__ __forceinline__ float cta_max(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  __syncthreads();  // red may still be read from a previous reduction
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float m = red[0];
#pragma unroll
  for (int i = 1; i < kFusedThreads / 32; ++i) m = fmaxf(m, red[i]);
  return m;
}

template <typename T, int D, class Seq>
__global__ void __launch_bounds__(kFusedThreads, 1)
quant_fused_kernel(const __grid_constant__ CUtensorMap tmap_q,
                   const __grid_constant__ CUtensorMap tmap_k,
                   const __grid_constant__ CUtensorMap tmap_v,
                   const __grid_constant__ Seq seq, const __grid_constant__ FusedQuantArgs a) {
  using L = FusedCfg<D>;
  constexpr int CPR = D / 8;                 // 16-byte chunks per row
  constexpr int RPP = kFusedThreads / CPR;   // rows per pass (32 for d = 128, 64 for d = 64)
  constexpr int NP = kPad / RPP;             // passes over a tile (4 or 2)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + L::kBarOff;
  float* redf = reinterpret_cast<float*>(smem + L::kRedOff);
  double* redd = reinterpret_cast<double*>(smem + L::kRedOff);
  const int tid = threadIdx.x;
  const int c = tid % CPR, rr = tid / CPR;   // this thread's chunk and first row
  cooperative_groups::grid_group grid = cooperative_groups::this_grid();

  if (tid == 0) {
    for (int s = 0; s < kFusedStages; ++s) mbar_init(bar0 + 8u * s, 1);
    fence_barrier_init();
    tma_prefetch_desc(&tmap_q);
    tma_prefetch_desc(&tmap_k);
    tma_prefetch_desc(&tmap_v);
  }
  __syncthreads();

  const int nQ = a.hq * a.nblk, nK = a.hkv * a.nblk;
  const int n1 = nQ + nK + (a.pv16 ? 0 : nK);  // phase 1 units
  const int n3 = 2 * nK;                        // phase 3 units
  uint32_t loads = 0;                           // tiles loaded by this CTA so far (all phases)
  bool ok = !watchdog_tripped();

  // unit -> (tensor 0/1/2 = Q/K/V, head, padded block)
  auto decode = [&](int phase, int u, int& tensor, int& h, int& pb) {
    if (phase == 1) {
      if (u < nQ) { tensor = 0; h = u / a.nblk; pb = u % a.nblk; return; }
      u -= nQ;
      tensor = u < nK ? 1 : 2;
      if (u >= nK) u -= nK;
    } else {
      tensor = u < nK ? 1 : 2;
      if (u >= nK) u -= nK;
    }
    h = u / a.nblk;
    pb = u % a.nblk;
  };
  auto issue = [&](int phase, int u, uint32_t slot) {  // one thread: TMA of unit u into a stage
    int tensor, h, pb;
    decode(phase, u, tensor, h, pb);
    const SeqPos sp = locate(seq, pb * kPad, 0, 0);
    const int row = (std::is_same<Seq, SeqVarlen>::value ? seq_base(seq, sp.b, 0, 1) : 0) +
                    (pb * kPad - sp.off);
    const int bco = std::is_same<Seq, SeqVarlen>::value ? 0 : sp.b;
    auto coord = [&](int d) { return a.dim_tok == d ? row : a.dim_head == d ? h : a.dim_batch == d ? bco : 0; };
    const CUtensorMap* m = tensor == 0 ? &tmap_q : tensor == 1 ? &tmap_k : &tmap_v;
    const uint32_t st = slot % kFusedStages;
    const uint32_t dst = sbase + st * L::kTile;
    mbar_arrive_expect_tx(bar0 + 8u * st, L::kTile);
#pragma unroll
    for (int bx = 0; bx < D / 64; ++bx)
      tma_load_4d(dst + bx * L::kBox, m, 64 * bx, coord(1), coord(2), coord(3), bar0 + 8u * st);
  };

  // ------------------------------------------------------------ per-unit work
  auto process = [&](int phase, int u, uint32_t slot) {
    int tensor, h, pb;
    decode(phase, u, tensor, h, pb);
    const SeqPos sp = locate(seq, pb * kPad, 0, 0);
    const int t0 = pb * kPad - sp.off;            // first token of the tile in its sequence
    const int nvalid = min(kPad, sp.n - t0);      // rows that belong to the sequence
    const uint32_t tile = sbase + (slot % kFusedStages) * L::kTile;
    float x[NP][8];
#pragma unroll
    for (int p = 0; p < NP; ++p) {
      const int r = rr + p * RPP;
      const uint4 v = lds16(tile + tile_off<D>(r, c));
      float f[8];
      unpack8<T>(v, f);
#pragma unroll
      for (int i = 0; i < 8; ++i) x[p][i] = (r < nvalid) ? f[i] : 0.0f;
    }
    const int64_t hb = static_cast<int64_t>(sp.b) * a.hkv + h;  // (sequence, kv head)

    if (phase == 1 && tensor == 1) {
      // ---- K: fp64 per-channel sums of this tile
      double s[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        s[i] = 0.0;
#pragma unroll
        for (int p = 0; p < NP; ++p) s[i] += static_cast<double>(x[p][i]);
      }
      // lanes with the same chunk: CPR apart within a warp, then across the warps
#pragma unroll
      for (int o = CPR; o < 32; o <<= 1)
#pragma unroll
        for (int i = 0; i < 8; ++i) s[i] += __shfl_xor_sync(0xffffffffu, s[i], o);
      __syncthreads();
      if ((tid & 31) < CPR)
#pragma unroll
        for (int i = 0; i < 8; ++i) redd[(tid >> 5) * D + c * 8 + i] = s[i];
      __syncthreads();
      if (tid < D) {
        double t = 0.0;
        for (int w = 0; w < kFusedThreads / 32; ++w) t += redd[w * D + tid];
        a.ksum[(static_cast<int64_t>(h) * a.nblk + pb) * D + tid] = t;
      }
      return;
    }
    if (phase == 1 && tensor == 2) {
      // ---- V: per-channel max |v| of this tile
      float m[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        m[i] = 0.0f;
#pragma unroll
        for (int p = 0; p < NP; ++p) m[i] = fmaxf(m[i], fabsf(x[p][i]));
      }
#pragma unroll
      for (int o = CPR; o < 32; o <<= 1)
#pragma unroll
        for (int i = 0; i < 8; ++i) m[i] = fmaxf(m[i], __shfl_xor_sync(0xffffffffu, m[i], o));
      __syncthreads();
      if ((tid & 31) < CPR)
#pragma unroll
        for (int i = 0; i < 8; ++i) redf[(tid >> 5) * D + c * 8 + i] = m[i];
      __syncthreads();
      if (tid < D) {
        float t = 0.0f;
        for (int w = 0; w < kFusedThreads / 32; ++w) t = fmaxf(t, redf[w * D + tid]);
        a.vpart[(static_cast<int64_t>(h) * a.nblk + pb) * D + tid] = t;
      }
      return;
    }
    if (tensor == 0 || tensor == 1) {
      // ---- Q (phase 1) or smoothed K (phase 3) -> INT8 blocks
      const bool isq = tensor == 0;
      if (!isq) {
        const float* mu = a.k_mean + hb * D + c * 8;
        float mv[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) mv[i] = mu[i];
#pragma unroll
        for (int p = 0; p < NP; ++p)
#pragma unroll
          for (int i = 0; i < 8; ++i)
            x[p][i] = (rr + p * RPP < nvalid) ? __fsub_rn(x[p][i], mv[i]) : 0.0f;
      }
      float rcp[NP];
      if (!a.fine) {
        // one scale per 128-token Q block, or per 64-token K block (rows of passes
        // p * RPP belong to K block p * RPP / 64)
        constexpr int KB = kBlkK / RPP;  // passes per 64-row K block (2 or 1)
        float bm[2] = {0.0f, 0.0f};
#pragma unroll
        for (int p = 0; p < NP; ++p) {
          float m = 0.0f;
#pragma unroll
          for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(x[p][i]));
          bm[p / KB] = fmaxf(bm[p / KB], m);  // K: each 64-row block; Q merges them below
        }
        if (isq) bm[0] = fmaxf(bm[0], bm[1]);
        const int nb = isq ? 1 : 2;
#pragma unroll
        for (int k2 = 0; k2 < 2; ++k2) {
          if (k2 >= nb) break;  // uniform over the CTA (the unit's tensor)
          const float amax = cta_max(bm[k2], redf);
          const float r = (amax > 0.0f) ? __fdiv_rn(127.0f, amax) : 0.0f;
#pragma unroll
          for (int p = 0; p < NP; ++p)
            if (isq || p / KB == k2) rcp[p] = r;
          if (tid == 0) {
            const float s = (amax > 0.0f) ? __fdiv_rn(amax, 127.0f) : 0.0f;
            if (isq) a.q_scale[static_cast<int64_t>(h) * a.nblk + pb] = s;
            else a.k_scale[static_cast<int64_t>(h) * (a.nblk * 2) + pb * 2 + k2] = s;
          }
        }
      } else if (isq) {
        // one scale per Q token: the CPR consecutive lanes holding a row reduce its max
#pragma unroll
        for (int p = 0; p < NP; ++p) {
          float m = 0.0f;
#pragma unroll
          for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(x[p][i]));
#pragma unroll
          for (int o = CPR / 2; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
          rcp[p] = (m > 0.0f) ? __fdiv_rn(127.0f, m) : 0.0f;
          if (c == 0)
            a.q_scale[static_cast<int64_t>(h) * seq.t_pad + pb * kPad + rr + p * RPP] =
                (m > 0.0f) ? __fdiv_rn(m, 127.0f) : 0.0f;
        }
      } else {
        // one scale per 32-token K block: pass p covers rows [p*RPP, (p+1)*RPP)
        constexpr int F = kBlkKFine;
        float bm[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int p = 0; p < NP; ++p) {
          float m = 0.0f;
#pragma unroll
          for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(x[p][i]));
          // rows of pass p lie in 32-row block (p*RPP + rr) / 32 (a select per block keeps
          // the array in registers)
          const int blk = (p * RPP + rr) / F;
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4) bm[k4] = blk == k4 ? fmaxf(bm[k4], m) : bm[k4];
        }
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) {
          const float amax = cta_max(bm[k4], redf);
          const float r = (amax > 0.0f) ? __fdiv_rn(127.0f, amax) : 0.0f;
#pragma unroll
          for (int p = 0; p < NP; ++p)
            if ((p * RPP + rr) / F == k4) rcp[p] = r;
          if (tid == 0)
            a.k_scale[static_cast<int64_t>(h) * (a.nblk * 4) + pb * 4 + k4] =
                (amax > 0.0f) ? __fdiv_rn(amax, 127.0f) : 0.0f;
        }
      }
      int8_t* dst = (isq ? a.q8 : a.k8) + (static_cast<int64_t>(h) * seq.t_pad + pb * kPad) * D + c * 8;
#pragma unroll
      for (int p = 0; p < NP; ++p) {
        const float r = rcp[p];
        uint2 o;
        o.x = pack_i8x4(quant_i8(x[p][0], r), quant_i8(x[p][1], r), quant_i8(x[p][2], r),
                        quant_i8(x[p][3], r));
        o.y = pack_i8x4(quant_i8(x[p][4], r), quant_i8(x[p][5], r), quant_i8(x[p][6], r),
                        quant_i8(x[p][7], r));
        *reinterpret_cast<uint2*>(dst + static_cast<int64_t>(rr + p * RPP) * D) = o;
      }
      return;
    }
    // ---- V (phase 3): e4m3 codes (or 16-bit values) written token-contiguous.  Thread
    // (chunk cv, token group tg) takes 8 channels x 4 consecutive tokens; a warp holds one
    // chunk and 32 token groups, so each channel row leaves as 128 (or 256) contiguous bytes.
    const int cv = tid >> 5, tg = tid & 31;  // 16 chunks x 32 groups (d = 128)
    if (cv < CPR) {
      // slot k holds token (k + tg) % 4 of the thread's four (read in that rotated order so
      // a warp's reads spread over the banks); the packed codes are rotated back to token
      // order with one funnel shift, so every index here is a compile-time one
      const int rot = tg & 3;
      float y[4][8];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int r = 4 * tg + ((k + rot) & 3);
        const uint4 v = lds16(tile + tile_off<D>(r, cv));
        float f[8];
        unpack8<T>(v, f);
#pragma unroll
        for (int i = 0; i < 8; ++i) y[k][i] = (r < nvalid) ? f[i] : 0.0f;
      }
      const int64_t row0 = static_cast<int64_t>(h) * D + cv * 8;
      if (!a.pv16) {
        const float* vm = a.vmax + hb * D + cv * 8;
        uint8_t* dst = reinterpret_cast<uint8_t*>(a.v8) + row0 * seq.t_pad + pb * kPad + 4 * tg;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float r = (vm[i] > 0.0f) ? __fdiv_rn(448.0f, vm[i]) : 0.0f;
          const uint32_t lo = e4m3x2(__fmul_rn(y[0][i], r), __fmul_rn(y[1][i], r));
          const uint32_t hi = e4m3x2(__fmul_rn(y[2][i], r), __fmul_rn(y[3][i], r));
          const uint32_t w = lo | (hi << 16);  // byte k = slot k
          *reinterpret_cast<uint32_t*>(dst + static_cast<int64_t>(i) * seq.t_pad) =
              __funnelshift_l(w, w, 8 * rot);  // byte (k + rot) % 4 = slot k
        }
      } else {
        T* dst = reinterpret_cast<T*>(a.v8) + row0 * seq.t_pad + pb * kPad + 4 * tg;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          uint64_t w = 0;  // 16-bit value k = slot k
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const T t = from_f32<T>(y[k][i]);
            w |= static_cast<uint64_t>(*reinterpret_cast<const uint16_t*>(&t)) << (16 * k);
          }
          if (rot != 0) w = (w << (16 * rot)) | (w >> (64 - 16 * rot));  // value (k + rot) % 4 = slot k
          *reinterpret_cast<uint64_t*>(dst + static_cast<int64_t>(i) * seq.t_pad) = w;
        }
      }
    }
  };

  // ------------------------------------------------------------ a phase over its units
  auto run_phase = [&](int phase, int count) {
    const int first = blockIdx.x, step = gridDim.x;
    const int mine = first < count ? (count - first + step - 1) / step : 0;
    if (tid == 0 && ok)
      for (int i = 0; i < min(mine, kFusedStages); ++i) issue(phase, first + i * step, loads + i);
    for (int i = 0; i < mine && ok; ++i) {
      const uint32_t slot = loads + i;
      ok = __syncthreads_and(mbar_wait(bar0 + 8u * (slot % kFusedStages),
                                       (slot / kFusedStages) & 1u, 0x501));
      if (!ok) break;
      process(phase, first + i * step, slot);
      __syncthreads();  // the stage has been read by every thread
      if (tid == 0 && i + kFusedStages < mine)
        issue(phase, first + (i + kFusedStages) * step, slot + kFusedStages);
    }
    loads += mine;
  };

  run_phase(1, n1);
  grid.sync();

  // ------------------------------------------------------------ phase 2: means, V scales
  {
    const int total = a.batch * a.hkv * D;
    for (int i = blockIdx.x * kFusedThreads + tid; i < total && ok; i += gridDim.x * kFusedThreads) {
      const int ch = i % D, hb = i / D, b = hb / a.hkv, h = hb % a.hkv;
      const int n = seq_len(seq, b);
      const int blk0 = seq_off(seq, b) / kPad;
      const int nb = (n + kPad - 1) / kPad;
      double s = 0.0;
      float m = 0.0f;
      for (int j = 0; j < nb; ++j) {
        const int64_t o = (static_cast<int64_t>(h) * a.nblk + blk0 + j) * D + ch;
        s += a.ksum[o];
        if (!a.pv16) m = fmaxf(m, a.vpart[o]);
      }
      a.k_mean[i] = (n > 0) ? __double2float_rn(__ddiv_rn(s, static_cast<double>(n))) : 0.0f;
      if (!a.pv16) {
        a.vmax[i] = m;
        a.v_scale[i] = (m > 0.0f) ? __fdiv_rn(m, 448.0f) : 0.0f;
      } else {
        a.v_scale[i] = 1.0f;
      }
    }
  }
  grid.sync();

  run_phase(3, n3);
}

}  // namespace sage
