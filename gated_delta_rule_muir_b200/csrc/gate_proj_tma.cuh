// Fused low-rank gate projection for bf16 inputs, fed by TMA (same operation as
// gate_proj.cuh: openai-hub article, section "五套门控被压进一个低秩投影";
// liuch.name post, second bullet).
//
//   h   = x W_down                            [N, 512], fp32 in TMEM
//   u_j = h[:, slice_j] U_j                   slices 64/64/128/128/128
//   log_alpha = log sigmoid(u_0); e, z, w, g = sigmoid(u_1..u_4)
//
// One CTA of 576 threads per 128-token tile (a TMA warp, an MMA warp and 16
// epilogue warps). Every operand tile that comes from
// global memory is a TMA box in 128-byte-swizzled shared memory (tma.cuh), so no
// thread stages the weights: bf16 values are exact and go to the tensor core as
// they are stored.
//   Down-projection: D in steps of 64. A stage is the x box (128 tokens x 64,
//     K-major) and the W_down rows (64 x 512 as eight 64-column boxes,
//     MN-major); two stages alternate, so the next stage's boxes land while the
//     current stage's two N = 256 MMAs run. One thread issues copies and MMAs.
//   Up-projections, by groups of h columns: {gates 0, 1} = h[:, 0:128), then
//     gate 2, 3, 4 = h[:, 128:256), [256:384), [384:512). The group's h columns
//     are drained by all threads into a bf16 hi/lo K-major tile (h keeps fp32
//     accuracy: two passes against the exact bf16 U), which frees those TMEM
//     columns; the gate's output columns then go in chunks of nch through two
//     TMEM buffers inside the freed columns, with the U boxes of the chunk after
//     next landing and the next chunk's MMA running while the threads apply the
//     activation to the current chunk and store it.
// Shared memory: two 80 KB stages (also the U chunk buffers) and the 64 KB h
// tile: 224 KB plus alignment.
#pragma once

#include "gate_proj.cuh"
#include "tma.cuh"

namespace muir {

struct GateTmaMaps {
  CUtensorMap x;      // [n][d], box 64 x 128
  CUtensorMap wd;     // [d][512], box 64 x 64
  CUtensorMap up[5];  // U_j [r_j][O_j], box 64 x r_j
};

constexpr uint32_t kGtStage = 80u * 1024u;        // x box (16 KB) + W_down rows (64 KB); or a U chunk
constexpr uint32_t kGtAh = 64u * 1024u;           // h group: 128 tokens x 128 ranks, bf16 hi and lo
constexpr uint32_t kGtSmem = 2u * kGtStage + kGtAh + 1024u;


// Hardware approximations of 2^x and log2(x) (relative error near 2^-22).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float lg2_approx(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Two sigmoids, 1 / d with d = 1 + 2^(-u log2 e), paired: one reciprocal serves
// both, 1/d1 = d2 / (d1 d2) and 1/d2 = d1 / (d1 d2). The exponent is capped at
// 57 so that d1 d2 stays finite; a sigmoid below 2^-57 comes out as 2^-57.
__device__ __forceinline__ float2 sigmoid2(float2 u) {
  const float2 a = __fmul2_rn(u, make_float2(-kLog2e, -kLog2e));
  const float2 d = __fadd2_rn(make_float2(ex2_approx(fminf(a.x, 57.f)), ex2_approx(fminf(a.y, 57.f))),
                              make_float2(1.f, 1.f));
  const float r = __fdividef(1.f, d.x * d.y);
  return __fmul2_rn(make_float2(d.y, d.x), make_float2(r, r));
}

// Activation and store of W consecutive output columns of one token row: log
// sigmoid into log_alpha (gate 0, fp32), sigmoid into the bf16 gates. The values
// come by reference to a fixed-size array so that they stay in registers.
template <int W>
__device__ __forceinline__ void emit_gate_w(const GateParams& p, int j, const float (&v)[W], int64_t o);

// Two log sigmoids, log sigmoid(u) = min(u, 0) - log1p(exp(-|u|)), paired where
// the operations allow; log1p(y) is formed as y * log(1 + y) / ((1 + y) - 1),
// which corrects the rounding of 1 + y (Goldberg, "What every computer scientist
// should know about floating-point arithmetic", 1991, Theorem 4), and as y where
// 1 + y rounds to 1.
__device__ __forceinline__ float2 log_sigmoid2(float2 u) {
  constexpr float kLn2 = 0.6931471805599453f;
  const float2 a = __fmul2_rn(make_float2(fabsf(u.x), fabsf(u.y)), make_float2(-kLog2e, -kLog2e));
  const float2 y = make_float2(ex2_approx(a.x), ex2_approx(a.y));
  const float2 w = __fadd2_rn(y, make_float2(1.f, 1.f));
  const float2 wm1 = __fadd2_rn(w, make_float2(-1.f, -1.f));
  const float2 l = __fmul2_rn(make_float2(lg2_approx(w.x), lg2_approx(w.y)), make_float2(kLn2, kLn2));
  const float l1x = w.x == 1.f ? y.x : y.x * __fdividef(l.x, wm1.x);
  const float l1y = w.y == 1.f ? y.y : y.y * __fdividef(l.y, wm1.y);
  return make_float2(fminf(u.x, 0.f) - l1x, fminf(u.y, 0.f) - l1y);
}

// Roles: warp 0 (one lane) issues the TMA copies, warp 1 (one lane) the MMAs,
// warps 2..17 are the epilogue: warp w reads TMEM lanes 32 (w % 4) .. + 31 (its
// token rows) and column group (w - 2) / 4 of every chunk. Hand-offs go through
// mbarriers only, so the epilogue never waits for the issuing threads except
// through the data:
//   full[s]      copies landed in stage s            (TMA -> MMA)
//   empty[s]     stage s read by its MMAs            (MMA commit -> TMA)
//   h_full       h complete in TMEM                  (MMA commit -> epilogue)
//   ah_full      the h group written to shared memory (16 epilogue warps -> MMA)
//   ah_empty     the h group's MMAs done             (MMA commit -> epilogue)
//   acc_full[b]  output buffer b computed            (MMA commit -> epilogue)
//   acc_empty[b] output buffer b read out            (16 epilogue warps -> MMA)
template <int W>
__device__ __forceinline__ void emit_gate_w(const GateParams& p, int j, const float (&v)[W], int64_t o) {
  if (j == 0) {
    float* dst = p.log_alpha + o;
#pragma unroll
    for (int q4 = 0; q4 < W; q4 += 4) {
      const float2 a = log_sigmoid2(make_float2(v[q4], v[q4 + 1]));
      const float2 b = log_sigmoid2(make_float2(v[q4 + 2], v[q4 + 3]));
      *reinterpret_cast<float4*>(dst + q4) = make_float4(a.x, a.y, b.x, b.y);
    }
  } else {
    __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.out[j]) + o;
#pragma unroll
    for (int q8 = 0; q8 < W; q8 += 8) {
      uint4 pk;
      __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&pk);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 sgm = sigmoid2(make_float2(v[q8 + 2 * e], v[q8 + 2 * e + 1]));
        h[e] = __floats2bfloat162_rn(sgm.x, sgm.y);
      }
      *reinterpret_cast<uint4*>(dst + q8) = pk;
    }
  }
}

constexpr int kGtEpiWarps = 16;
constexpr int kGtThreads = 32 * (2 + kGtEpiWarps);

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// The h groups and the gates of each: gates 0 and 1 share h columns [0, 128);
// gate 2, 3, 4 take [128, 256), [256, 384), [384, 512). A gate's output goes in
// chunks of nch columns through two TMEM buffers at [0, nch) and [nch, 2 nch),
// inside h columns that are already drained.
__host__ __device__ constexpr int gt_group_of(int j) { return j < 2 ? 0 : j - 1; }
__host__ __device__ constexpr int gt_nch(int j) { return j < 2 ? 64 : j < 4 ? 128 : 256; }
__host__ __device__ constexpr int gt_rank0(int j) { return j == 1 ? 64 : 0; }  // first rank inside the h tile

__global__ void __launch_bounds__(kGtThreads, 1) gate_proj_tma_kernel(const __grid_constant__ GateTmaMaps m,
                                                                       GateParams p) {
  extern __shared__ __align__(1024) uint8_t sm[];
  __shared__ uint64_t full[2], empty[2], h_full, ah_full, ah_empty, acc_full[2], acc_empty[2];
  __shared__ uint32_t tslot;
  const int tid = threadIdx.x, warp = tid >> 5, lane_id = tid & 31;
  const int64_t row0 = (int64_t)blockIdx.x * 128;
  const uint32_t base = (smem_u32(sm) + 1023u) & ~1023u;
  const uint32_t ah = base + 2u * kGtStage;  // h group: hi boxes at ah, ah + 16 KB; lo at ah + 32 KB, + 48 KB
  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], kGtEpiWarps);
    }
    mbar_init(&h_full, 1);
    mbar_init(&ah_full, kGtEpiWarps);
    mbar_init(&ah_empty, 1);
    tma_prefetch_desc(&m.x);
    tma_prefetch_desc(&m.wd);
  }
  if (warp == 0) tmem_alloc(&tslot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tslot;
  const int nk = p.d / 64;
  auto O_of = [&](int j) { return (j == 2 || j == 3) ? p.ov : p.ok; };

  if (warp == 0) {
    // ---- TMA producer: the down-projection stages, then the U chunks -------
    if (lane_id == 0) {
      // phase bookkeeping in registers (bit s: parity of stage s's next wait;
      // a dynamically indexed array would live in local memory)
      uint32_t used = 0, eph = 0;  // used: bit s once stage s has been filled
      bool ok = true;
      auto acquire = [&](int s) {  // wait until stage s is free
        if ((used >> s) & 1u) {
          ok = mbar_wait(&empty[s], (eph >> s) & 1u);
          eph ^= 1u << s;
        }
        used |= 1u << s;
        return ok;
      };
      int i = 0;  // stage counter
      for (int ks = 0; ks < nk && ok; ++ks, ++i) {
        const int s = i & 1;
        if (!acquire(s)) break;
        const uint32_t st = base + (uint32_t)s * kGtStage;
        mbar_expect_tx(&full[s], kGtStage);
        tma_load_2d(st, &m.x, 64 * ks, (int)row0, &full[s]);
        for (int b = 0; b < 8; ++b) tma_load_2d(st + 16384u + (uint32_t)b * 8192u, &m.wd, 64 * b, 64 * ks, &full[s]);
      }
      for (int j = 0; j < 5 && ok; ++j) {
        const int r = gate_rank(j), nch = gt_nch(j), nchunk = O_of(j) / nch;
        const uint32_t ubytes = (uint32_t)r * 128u;  // one 64-column U box
        for (int c = 0; c < nchunk && ok; ++c, ++i) {
          const int s = i & 1;
          if (!acquire(s)) break;
          const uint32_t st = base + (uint32_t)s * kGtStage;
          mbar_expect_tx(&full[s], ubytes * (uint32_t)(nch / 64));
          for (int b = 0; b < nch / 64; ++b)
            tma_load_2d(st + (uint32_t)b * ubytes, &m.up[j], c * nch + 64 * b, 0, &full[s]);
        }
      }
    }
  } else if (warp == 1) {
    // ---- MMA issuer ----------------------------------------------------------
    if (lane_id == 0) {
      uint32_t fph = 0;               // bit s: parity of stage s's next full wait
      uint32_t bused = 0, bph = 0;    // bit b: buffer b has been filled / parity of its next drain wait
      bool ok = true;
      int i = 0;
      const uint32_t id1 = idesc_bf16(128, 256, 0, 1);
      for (int ks = 0; ks < nk && ok; ++ks, ++i) {
        const int s = i & 1;
        ok = mbar_wait(&full[s], (fph >> s) & 1u);
        fph ^= 1u << s;
        if (!ok) break;
        tc_fence_after();
        const uint32_t st = base + (uint32_t)s * kGtStage;
        for (int k16 = 0; k16 < 4; ++k16) {
          const uint64_t ad = sdesc_sw128(st + (uint32_t)k16 * 32u, 16u, 1024u);
          for (int hh = 0; hh < 2; ++hh) {
            const uint64_t bd =
                sdesc_sw128(st + 16384u + (uint32_t)hh * 4u * 8192u + (uint32_t)k16 * 2048u, 8192u, 1024u);
            mma_bf16(tmem + (uint32_t)hh * 256u, ad, bd, id1, (ks > 0 || k16 > 0) ? 1u : 0u);
          }
        }
        mma_commit(&empty[s]);
      }
      if (ok) mma_commit(&h_full);
      // wait until the given buffer's last contents have been read out (a wait on
      // a phase that has already completed returns at once, so asking twice is fine)
      auto buffer_free = [&](int b) {
        if ((bused >> b) & 1u) return mbar_wait(&acc_empty[b], (bph >> b) & 1u);
        return true;
      };
      int q = 0;  // output chunk counter (buffer q & 1)
      for (int g = 0; g < 4 && ok; ++g) {
        ok = mbar_wait(&ah_full, (uint32_t)g & 1u);  // the group's h columns are in shared memory
        if (!ok) break;
        tc_fence_after();
        for (int j = g == 0 ? 0 : g + 1; j <= (g == 0 ? 1 : g + 1) && ok; ++j) {
          const int r = gate_rank(j), nch = gt_nch(j), nchunk = O_of(j) / nch, rank0 = gt_rank0(j);
          const uint32_t ubytes = (uint32_t)r * 128u;
          const uint32_t id = idesc_bf16(128, nch, 0, 1);
          // a new column layout: both buffers must have been read out
          ok = buffer_free(0) && buffer_free(1);
          for (int c = 0; c < nchunk && ok; ++c, ++i, ++q) {
            const int s = i & 1, b = q & 1;
            ok = mbar_wait(&full[s], (fph >> s) & 1u);
            fph ^= 1u << s;
            ok = ok && buffer_free(b);
            if (!ok) break;
            tc_fence_after();
            const uint32_t st = base + (uint32_t)s * kGtStage;
            const uint32_t acc = tmem + (uint32_t)(b * nch);
            for (int k16 = 0; k16 < r / 16; ++k16) {
              const int kr = rank0 + 16 * k16;
              const uint32_t ao = (uint32_t)(kr >> 6) * 16384u + (uint32_t)((kr & 63) * 2);
              const uint64_t bd = sdesc_sw128(st + (uint32_t)k16 * 2048u, ubytes, 1024u);
              mma_bf16(acc, sdesc_sw128(ah + ao, 16u, 1024u), bd, id, k16 > 0 ? 1u : 0u);
              mma_bf16(acc, sdesc_sw128(ah + 32768u + ao, 16u, 1024u), bd, id, 1u);
            }
            mma_commit(&empty[s]);
            mma_commit(&acc_full[b]);
            // bit b of bph: parity of the drain of b's latest fill (fill k is drained in phase k)
            if ((bused >> b) & 1u) bph ^= 1u << b;
            bused |= 1u << b;
          }
        }
        if (ok) mma_commit(&ah_empty);  // the group's MMAs done: the h tile may be rewritten
      }
      // the last commit has arrived once every MMA has completed: nothing is left in flight
      if (ok) mbar_wait(&ah_empty, 1u);
    }
  } else {
    // ---- epilogue warps --------------------------------------------------------
    const int e = warp - 2;
    const int grp = e >> 2;                    // column group 0..3
    const uint32_t lane = tmem_lane_base(warp);  // TMEM lanes 32 (warp % 4) ..
    const int t = ((warp & 3) << 5) | lane_id;   // token row of this thread
    const bool on = row0 + t < p.n;
    bool ok = mbar_wait(&h_full, 0u);
    tc_fence_after();
    int q = 0;
    uint32_t aph = 0;  // bit b: parity of buffer b's next full wait
    for (int g = 0; g < 4 && ok; ++g) {
      if (g > 0) {
        ok = mbar_wait(&ah_empty, (uint32_t)(g - 1) & 1u);
        if (!ok) break;
        tc_fence_after();
      }
      // h columns [128 g, 128 g + 128) -> the h tile (bf16 hi/lo, K-major, 128-byte swizzle)
      {
        const int c = grp * 32;
        float v[32];
        tmem_ld32(tmem + lane + (uint32_t)(128 * g + c), v);
#pragma unroll
        for (int hf = 0; hf < 4; ++hf) {
          float x8[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) x8[k] = v[8 * hf + k];
          uint4 hi, lo;
          split8(x8, hi, lo);
          const int cc = c + 8 * hf;
          const uint32_t off =
              (uint32_t)(cc >> 6) * 16384u + (uint32_t)t * 128u + (uint32_t)((((cc & 63) >> 3) ^ (t & 7)) * 16);
          sts128(ah + off, hi);
          sts128(ah + 32768u + off, lo);
        }
        fence_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane_id == 0) mbar_arrive(&ah_full);
      }
      for (int j = g == 0 ? 0 : g + 1; j <= (g == 0 ? 1 : g + 1) && ok; ++j) {
        const int nch = gt_nch(j), O = O_of(j), nchunk = O / nch, W = nch / 4;
        for (int c = 0; c < nchunk; ++c, ++q) {
          const int b = q & 1;
          ok = mbar_wait(&acc_full[b], (aph >> b) & 1u);
          aph ^= 1u << b;
          if (!ok) break;
          tc_fence_after();
          const uint32_t acc = tmem + lane + (uint32_t)(b * nch + grp * W);
          const int64_t o = (row0 + t) * O + (int64_t)c * nch + grp * W;
          if (W == 16) {
            float v[16];
            tmem_ld16(acc, v);
            tc_fence_before();
            __syncwarp();
            if (lane_id == 0) mbar_arrive(&acc_empty[b]);
            if (on) emit_gate_w<16>(p, j, v, o);
          } else {
            for (int h32 = 0; h32 < W; h32 += 32) {
              float v[32];
              tmem_ld32(acc + (uint32_t)h32, v);
              if (h32 + 32 >= W) {  // the buffer has been read: hand it back before the math
                tc_fence_before();
                __syncwarp();
                if (lane_id == 0) mbar_arrive(&acc_empty[b]);
              }
              if (on) emit_gate_w<32>(p, j, v, o + h32);
            }
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

}  // namespace muir
