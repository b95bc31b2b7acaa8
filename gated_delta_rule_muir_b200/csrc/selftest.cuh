// Diagnostic GEMM exercising the tcgen05 operand layouts of tc.cuh:
// D[M=128, N] = A[128, K] * B[K, N] with fp32 row-major A and B in global
// memory, staged K-major or MN-major, 1-pass or 3-pass bf16. One CTA.
#pragma once

#include "tc.cuh"
#include "tma.cuh"

namespace muir {

__global__ void __launch_bounds__(128) selftest_gemm_kernel(const float* __restrict__ A, const float* __restrict__ B,
                                                            float* __restrict__ D, int N, int K, int a_mn, int b_mn,
                                                            int nsplit) {
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ uint64_t bar;
  __shared__ uint32_t tmem_base;
  const int tid = threadIdx.x, warp = tid >> 5;
  const uint32_t base = smem_u32(smem);
  const uint32_t a_bytes = 128u * K * 2u, b_bytes = (uint32_t)N * K * 2u;
  Tile ta{base, base + a_bytes, 128u, (uint32_t)K * 16u};
  Tile tb{base + 2 * a_bytes, base + 2 * a_bytes + b_bytes, 128u, (uint32_t)K * 16u};
  if (warp == 0) tmem_alloc(&tmem_base, N <= 32 ? 32 : (N <= 64 ? 64 : (N <= 128 ? 128 : 256)));
  if (tid == 0) mbar_init(&bar, 1);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;

  // Operand modes: bit 0 = major (0 K-major, 1 MN-major); bit 1 = the tile is
  // written in the other arrangement and read through transposed().
  const int a_major = a_mn & 1, b_major = b_mn & 1;
  Tile ta_w = ta, tb_w = tb;
  if (a_mn & 2) ta_w.sbo = 128u * 16u;     // arrangement stride over the 128 rows/cols of A
  if (b_mn & 2) tb_w.sbo = (uint32_t)N * 16u;
  // A: element (m, k) = A[m*K + k]
  for (int idx = tid; idx < 128 * (K / 8); idx += 128) {
    float x[8];
    if (a_mn == 0 || a_mn == 2) {  // rows m, 8 consecutive k
      const int m = idx / (K / 8), k8 = (idx % (K / 8)) * 8;
#pragma unroll
      for (int e = 0; e < 8; ++e) x[e] = A[m * K + k8 + e];
      if (a_mn == 0) put_k(ta_w, m, k8, x);
      else put_mn(ta_w, m, k8, x);
    } else {                        // rows k, 8 consecutive m
      const int k = idx / 16, m8 = (idx % 16) * 8;
#pragma unroll
      for (int e = 0; e < 8; ++e) x[e] = A[(m8 + e) * K + k];
      if (a_mn == 1) put_mn(ta_w, k, m8, x);
      else put_k(ta_w, k, m8, x);
    }
  }
  // B: element (k, n) = B[k*N + n]
  for (int idx = tid; idx < N * (K / 8); idx += 128) {
    float x[8];
    if (b_mn == 0 || b_mn == 2) {  // rows n, 8 consecutive k
      const int n = idx / (K / 8), k8 = (idx % (K / 8)) * 8;
#pragma unroll
      for (int e = 0; e < 8; ++e) x[e] = B[(k8 + e) * N + n];
      if (b_mn == 0) put_k(tb_w, n, k8, x);
      else put_mn(tb_w, n, k8, x);
    } else {                        // rows k, 8 consecutive n
      const int k = idx / (N / 8), n8 = (idx % (N / 8)) * 8;
#pragma unroll
      for (int e = 0; e < 8; ++e) x[e] = B[k * N + n8 + e];
      if (b_mn == 1) put_mn(tb_w, k, n8, x);
      else put_k(tb_w, k, n8, x);
    }
  }
  if (a_mn & 2) ta = transposed(ta_w);
  if (b_mn & 2) tb = transposed(tb_w);
  MmaSync drv{&bar, 0u, true};
  const uint32_t id = idesc_bf16(128, N, a_major, b_major);
  drv.run([&] { mma_tiles(tmem, ta, tb, K / 16, id, nsplit, false); });
  if (drv.ok) {
    for (int c = 0; c < N; c += 16) {
      float v[16];
      tmem_ld16(tmem + tmem_lane_base(warp) + c, v);
#pragma unroll
      for (int i = 0; i < 16; ++i) D[tid * N + c + i] = v[i];
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, N <= 32 ? 32 : (N <= 64 ? 64 : (N <= 128 ? 128 : 256)));
}

// Exercises the give-up path of the bounded wait. One warp initialises an
// mbarrier (count 1) in its own shared memory; with `arrive` set, thread 0
// arrives first so the phase completes, otherwise nothing ever arrives. Thread
// 0 then waits for phase 0 through mbar_wait_for with limit_ns. No copy or MMA
// is in flight at any time, so the kernel ends cleanly either way; a wait that
// ran out is recorded in the status word. out[0] = 1 if the wait saw the phase
// complete, 0 if it gave up.
__global__ void __launch_bounds__(32) selftest_wait_kernel(uint64_t limit_ns, int arrive, int* out) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    if (arrive) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&bar)) : "memory");
    out[0] = mbar_wait_for(&bar, 0u, limit_ns) ? 1 : 0;
  }
}

// D[128, N] = A[128, K] B[K, N], bf16 A (row-major: the K-major operand) and B
// (row-major [K][N]: the MN-major operand), through 128-byte-swizzled shared
// memory filled by TMA boxes (mode 1) or by the threads in the same layout
// (mode 0). Mode 2 has the threads store A transposed, as the MN-major operand:
// rows = K, 64-column boxes along M (the layout of a token-major tile read as
// the A operand of a product over tokens). K in {64, 128}; N in {64, 128, 256}.
// One CTA of 128 threads.
__global__ void __launch_bounds__(128) selftest_sw128_kernel(const __grid_constant__ CUtensorMap ta,
                                                             const __grid_constant__ CUtensorMap tb,
                                                             const __nv_bfloat16* __restrict__ A,
                                                             const __nv_bfloat16* __restrict__ B, float* __restrict__ D,
                                                             int N, int K, int mode) {
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ uint64_t bar, bar_cp;
  __shared__ uint32_t tslot;
  const int tid = threadIdx.x, warp = tid >> 5;
  const uint32_t base = (smem_u32(smem) + 1023u) & ~1023u;
  const uint32_t bbase = base + (uint32_t)(K / 64) * 16384u;
  const uint32_t ncols = N <= 32 ? 32u : N <= 64 ? 64u : N <= 128 ? 128u : 256u;
  if (warp == 0) tmem_alloc(&tslot, ncols);
  if (tid == 0) {
    mbar_init(&bar, 1);
    mbar_init(&bar_cp, 1);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tslot;
  bool ok = true;
  if (mode == 1) {
    if (tid == 0) {
      mbar_expect_tx(&bar_cp, (uint32_t)(K / 64) * 16384u + (uint32_t)(N / 64) * (uint32_t)K * 128u);
      for (int a = 0; a < K / 64; ++a) tma_load_2d(base + a * 16384u, &ta, 64 * a, 0, &bar_cp);
      for (int n = 0; n < N / 64; ++n) tma_load_2d(bbase + (uint32_t)n * K * 128u, &tb, 64 * n, 0, &bar_cp);
    }
    ok = __syncthreads_and(mbar_wait(&bar_cp, 0) ? 1 : 0) != 0;
  } else {
    if (mode == 2) {
      for (int idx = tid; idx < K * 16; idx += 128) {  // row k of A^T: 16 pieces of 8 values of m
        const int k = idx / 16, c = idx % 16;
        __align__(16) __nv_bfloat16 e[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) e[j] = A[(int64_t)(8 * c + j) * K + k];
        sts128(base + (uint32_t)(c / 8) * K * 128u + (uint32_t)k * 128u + (uint32_t)(((c % 8) ^ (k & 7)) * 16),
               *reinterpret_cast<const uint4*>(e));
      }
    } else {
      for (int idx = tid; idx < 128 * (K / 8); idx += 128) {
        const int m = idx / (K / 8), c = idx % (K / 8);
        const uint4 v = *reinterpret_cast<const uint4*>(A + (int64_t)m * K + 8 * c);
        sts128(base + (uint32_t)(c / 8) * 16384u + (uint32_t)m * 128u + (uint32_t)(((c % 8) ^ (m & 7)) * 16), v);
      }
    }
    for (int idx = tid; idx < K * (N / 8); idx += 128) {
      const int k = idx / (N / 8), c = idx % (N / 8);
      const uint4 v = *reinterpret_cast<const uint4*>(B + (int64_t)k * N + 8 * c);
      sts128(bbase + (uint32_t)(c / 8) * K * 128u + (uint32_t)k * 128u + (uint32_t)(((c % 8) ^ (k & 7)) * 16), v);
    }
    fence_async_smem();
    __syncthreads();
  }
  if (ok && tid == 0) {
    tc_fence_after();
    const uint32_t id = idesc_bf16(128, N, mode == 2 ? 1 : 0, 1);
    for (int ks = 0; ks < K / 16; ++ks) {
      const uint64_t ad = mode == 2 ? sdesc_sw128(base + (uint32_t)ks * 2048u, (uint32_t)K * 128u, 1024u)
                                    : sdesc_sw128(base + (uint32_t)(ks / 4) * 16384u + (uint32_t)(ks % 4) * 32u, 16u, 1024u);
      const uint64_t bd = sdesc_sw128(bbase + (uint32_t)ks * 2048u, (uint32_t)K * 128u, 1024u);
      mma_bf16(tmem, ad, bd, id, ks > 0 ? 1u : 0u);
    }
    mma_commit(&bar);
  }
  if (ok) ok = __syncthreads_and(mbar_wait(&bar, 0) ? 1 : 0) != 0;
  tc_fence_after();
  if (ok) {
    for (int c = 0; c < N; c += 16) {
      float v[16];
      tmem_ld16(tmem + tmem_lane_base(warp) + c, v);
#pragma unroll
      for (int i = 0; i < 16; ++i) D[tid * N + c + i] = v[i];
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, ncols);
}

}  // namespace muir
