// debug_qk.cuh - test hook: exact int32 S = Q8 K8^T tiles through the same
// TMA + tcgen05.mma kind::i8 + TMEM path as the attention kernel.
// (vibecrowd repo page "thu-ml--sageattention", How it works: INT8 QK^T.)
#pragma once

#include "sage_device.cuh"

namespace sage {

template <int D>
__global__ void __launch_bounds__(128, 1)
debug_qk_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                int q_row0, int k_row0, int p_len, int32_t* __restrict__ s_out) {
  constexpr int kTile = kBlkQ * D;
  constexpr uint32_t kSwizzle = (D == 128) ? 2u : 4u;
  constexpr uint32_t kSbo = 8u * D;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sq = smem_u32(smem), sk = sq + kTile;
  const uint32_t bar_load = sk + kTile, bar_mma = bar_load + 8;
  uint32_t* slot = reinterpret_cast<uint32_t*>(smem + 2 * kTile + 16);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = blockIdx.x, kt = blockIdx.y;

  if (threadIdx.x == 0) {
    mbar_init(bar_load, 1);
    mbar_init(bar_mma, 1);
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(slot), 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *slot;

  if (threadIdx.x == 0 && !watchdog_tripped()) {
    mbar_arrive_expect_tx(bar_load, 2 * kTile);
    tma_load_2d(sq, &tmap_q, 0, q_row0 + qt * kBlkQ, bar_load);
    tma_load_2d(sk, &tmap_k, 0, k_row0 + kt * kBlkQ, bar_load);
    if (mbar_wait(bar_load, 0, 0x401)) {
      tc_fence_after();
#pragma unroll
      for (int s = 0; s < D / 32; ++s)
        mma_i8_ss(tmem, sdesc_kmajor(sq + 32u * s, kSbo, kSwizzle),
                  sdesc_kmajor(sk + 32u * s, kSbo, kSwizzle), idesc_i8(128, 128), s > 0 ? 1u : 0u);
    }
    tc_commit(bar_mma);
  }
  __syncwarp();
  const bool ok = __all_sync(0xffffffffu, mbar_wait(bar_mma, 0, 0x402));
  tc_fence_after();
  if (ok) {
    const int row = warp * 32 + lane;
    int32_t* dst = s_out + static_cast<int64_t>(qt * kBlkQ + row) * p_len + kt * kBlkQ;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint32_t r[32];
      tmem_ld32(tmem + (static_cast<uint32_t>(warp * 32) << 16) + 32u * c, r);
      tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < 32; i += 4)
        *reinterpret_cast<int4*>(dst + 32 * c + i) =
            make_int4(static_cast<int>(r[i]), static_cast<int>(r[i + 1]),
                      static_cast<int>(r[i + 2]), static_cast<int>(r[i + 3]));
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) {
    __syncwarp();
    tmem_dealloc(tmem, 128);
  }
}

// Failure-path self-test: thread 0 waits on an mbarrier phase that never completes
// (its count is 1 and nothing arrives), polling as the kernels' bounded waits do, and
// records a timeout in the watchdog word once limit_ns have passed.
__global__ void __launch_bounds__(32) watchdog_selftest_kernel(uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  const uint32_t b = smem_u32(&bar);
  mbar_init(b, 1);
  fence_barrier_init();
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(b, 0)) {
    if (global_timer_ns() - t0 > limit_ns) {
      watchdog_trip(0x7E57);
      return;
    }
  }
}

}  // namespace sage
