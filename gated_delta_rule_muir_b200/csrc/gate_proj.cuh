// Fused low-rank gate projection: the five gate tensors of the operator from
// the layer input, with one shared down-projection.
//
// Source: openai-hub article "Google Research 提出 Muir：25MB 固定状态跑完千万 Token",
// section "五套门控被压进一个低秩投影" (table of gate ranks), and the liuch.name
// post, second bullet: decay, erase, output, write and dynamic-read gates share
// one down-projection of total rank 512, then each has its own up-projection,
// with ranks 64, 64, 128, 128, 128 in that order.
//
//   h     = x W_down                      [N, 512], fp32 accumulation
//   u_j   = h[:, slice_j] U_j             slice_j: [0,64) [64,128) [128,256) [256,384) [384,512)
//   log_alpha = log sigmoid(u_decay), e = sigmoid(u_erase), z = sigmoid(u_out),
//   w = sigmoid(u_write), g = sigmoid(u_read)
//
// One CTA of 256 threads per 128-token tile. h stays on chip: its 128 x 512
// fp32 tile fills TMEM. The down-projection runs over D in 64-wide K steps (x
// tile K-major, W_down tile MN-major, two N = 256 MMAs per step; one bf16 pass
// for bf16 inputs, whose products are exact and whose packed values are stored
// as they are, three hi/lo passes for fp32). Then gate by gate the rank slice of
// h is drained to shared memory as a bf16 hi/lo K-major operand and multiplied
// by column chunks of U_j (h's hi and lo parts, so h keeps fp32 accuracy: 2
// passes against an exact bf16 U, 3 against fp32) into TMEM columns whose
// slices have already been drained; the activation is applied on the way out.
#pragma once

#include "chunk.cuh"

namespace muir {

struct GateParams {
  const void* x;      // [n][d]
  const void* wd;     // [d][512]
  const void* up[5];  // U_decay, U_erase [64][ok]; U_out, U_write [128][ov]; U_read [128][ok]
  float* log_alpha;   // [n][ok]
  void* out[5];       // out[1..4] = e [n][ok], z [n][ov], w [n][ov], g [n][ok]; out[0] unused
  int64_t n;          // tokens
  int d;              // d_model, a multiple of 64
  int ok, ov;         // H d_k and H d_v, multiples of 256
};

// rank and first column of gate j's slice of h: 64/64/128/128/128 from 0, 64, 128, 256, 384
__host__ __device__ constexpr int gate_rank(int j) { return j < 2 ? 64 : 128; }
__host__ __device__ constexpr int gate_off(int j) { return j == 0 ? 0 : j == 1 ? 64 : 128 * (j - 1); }
constexpr uint32_t kGateSmem = 192u * 1024u;

// The fast exponential and division intrinsics (a few ulp): the epilogue applies
// one activation per output element, which dominates the kernel's instruction
// count with the correctly rounded forms. For u << 0 the denominator overflows
// to +inf and the quotient is 0.
__device__ __forceinline__ float gate_sigmoid(float u) { return __fdividef(1.f, 1.f + __expf(-u)); }
// log(sigmoid(u)) = min(u, 0) - log(1 + exp(-|u|)), finite for every finite u;
// log1pf keeps its accuracy near 0 (slow-decay rows)
__device__ __forceinline__ float gate_log_sigmoid(float u) { return fminf(u, 0.f) - log1pf(__expf(-fabsf(u))); }

template <typename T, int NS1>
__global__ void __launch_bounds__(256, 1) gate_proj_kernel(GateParams p) {
  extern __shared__ __align__(128) uint8_t sm[];
  __shared__ uint64_t bar;
  __shared__ uint32_t tslot;
  constexpr int NT = 256, KC = 64;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int64_t row0 = (int64_t)blockIdx.x * 128;
  const uint32_t base = smem_u32(sm);
  TcCta cta;
  cta.init(&tslot, &bar, 512);
  MmaSync drv{&bar, 0u, true};

  // ---- h = x W_down into TMEM columns [0, 512)
  const Tile X{base, base + 16384u, 128u, KC * 16u};                // 128 tokens x 64, K-major
  const Tile Wt{base + 32768u, base + 32768u + 65536u, 128u, KC * 16u};  // 64 (K) x 512 (N), MN-major
  const T* xp = static_cast<const T*>(p.x);
  const T* wd = static_cast<const T*>(p.wd);
  // A K step's loads go out at once (into px, pw); the next step's while the
  // current step's MMAs run.
  constexpr int XP = 128 * (KC / 8) / NT, WP = KC * (512 / 8) / NT;  // pieces per thread
  Pack8<T> px[XP], pw[WP];
  auto load_xw = [&](int k0) {
#pragma unroll
    for (int m = 0; m < XP; ++m) {
      int r, c8;
      piece_of<KC / 8>(tid + m * NT, r, c8);
      if (row0 + r < p.n) px[m].ld(xp + (row0 + r) * p.d + k0 + c8);
    }
#pragma unroll
    for (int m = 0; m < WP; ++m) {
      int k, n8;
      piece_of<512 / 8>(tid + m * NT, k, n8);
      pw[m].ld(wd + (int64_t)(k0 + k) * 512 + n8);
    }
  };
  load_xw(0);
  for (int k0 = 0; k0 < p.d && drv.ok; k0 += KC) {
#pragma unroll
    for (int m = 0; m < XP; ++m) {
      int r, c8;
      piece_of<KC / 8>(tid + m * NT, r, c8);
      if constexpr (sizeof(T) == 2) {  // exact in bf16: the packed values are the hi plane
        put_k_raw(X, r, c8, row0 + r < p.n ? px[m].u : make_uint4(0, 0, 0, 0));
      } else {
        float v[8];
        if (row0 + r < p.n) {
          px[m].get(v);
        } else {  // rows past the last token
#pragma unroll
          for (int j = 0; j < 8; ++j) v[j] = 0.f;
        }
        put_k(X, r, c8, v);
      }
    }
#pragma unroll
    for (int m = 0; m < WP; ++m) {
      int k, n8;
      piece_of<512 / 8>(tid + m * NT, k, n8);
      if constexpr (sizeof(T) == 2) {
        put_mn_raw(Wt, k, n8, pw[m].u);
      } else {
        float v[8];
        pw[m].get(v);
        put_mn(Wt, k, n8, v);
      }
    }
    drv.run_overlap(
        [&] {
          const uint32_t id = idesc_bf16(128, 256, 0, 1);
          mma_tiles(cta.tmem + 0, X, Wt, KC / 16, id, NS1, k0 > 0);
          const Tile W2{Wt.hi + 32u * Wt.sbo, Wt.lo + 32u * Wt.sbo, Wt.lbo, Wt.sbo};  // columns 256..511
          mma_tiles(cta.tmem + 256, X, W2, KC / 16, id, NS1, k0 > 0);
        },
        [&] {
          if (k0 + KC < p.d) load_xw(k0 + KC);
        });
  }

  // ---- gate by gate: u_j = h_j U_j, activated
  const Tile Ah{base, base + 32768u, 128u, 128u * 16u};               // h_j: 128 tokens x r_j, K-major
  const Tile Ub{base + 65536u, base + 131072u, 128u, 128u * 16u};     // U_j chunk: r_j (K) x nch (N), MN-major
  const uint32_t lane = tmem_lane_base(warp);
  const int t = tid & 127, wg = tid >> 7;  // TMEM row (token); warpgroups take alternate 16-column chunks
  const bool on = row0 + t < p.n;
  constexpr int UP = 128 * (256 / 8) / NT;  // U pieces per thread at most (r = 128, nch = 256)
  constexpr int kUpPasses = sizeof(T) == 2 ? 2 : 3;
  Pack8<T> pu[UP];
  for (int j = 0; j < 5 && drv.ok; ++j) {
    const int r = gate_rank(j), off = gate_off(j);
    const int O = (j == 2 || j == 3) ? p.ov : p.ok;
    // columns [0, off + r) of TMEM are free once h_j is drained; chunks use [0, nch)
    const int nch = j == 0 ? 64 : j == 1 ? 128 : 256;
    for (int c = wg * 16; c < r; c += 32) {
      float v[16];
      tmem_ld16(cta.tmem + lane + off + c, v);
      float a8[8], b8[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) { a8[e] = v[e]; b8[e] = v[8 + e]; }
      put_k(Ah, t, c, a8);
      put_k(Ah, t, c + 8, b8);
    }
    // U_j chunk n0: all of a thread's loads go out at once (into pu), the next
    // chunk's while the current chunk's MMA runs
    const T* U = static_cast<const T*>(p.up[j]);
    const int np = r * (nch / 8);
    auto load_u = [&](int n0) {
#pragma unroll
      for (int m = 0; m < UP; ++m) {
        const int x = tid + m * NT;
        if (x < np) {
          int k, n8;
          piece_of_rt(x, nch / 8, k, n8);
          pu[m].ld(U + (int64_t)k * O + n0 + n8);
        }
      }
    };
    load_u(0);
    for (int n0 = 0; n0 < O && drv.ok; n0 += nch) {
#pragma unroll
      for (int m = 0; m < UP; ++m) {
        const int x = tid + m * NT;
        if (x < np) {
          int k, n8;
          piece_of_rt(x, nch / 8, k, n8);
          if constexpr (sizeof(T) == 2) {
            put_mn_raw(Ub, k, n8, pu[m].u);
          } else {
            float v[8];
            pu[m].get(v);
            put_mn(Ub, k, n8, v);
          }
        }
      }
      // bf16 U is exact: h's hi and lo parts times U's hi plane (2 passes); fp32 U: 3 passes
      drv.run_overlap([&] { mma_tiles(cta.tmem, Ah, Ub, r / 16, idesc_bf16(128, nch, 0, 1), kUpPasses, false); },
                      [&] {
                        if (n0 + nch < O) load_u(n0 + nch);
                      });
      for (int c = wg * 16; c < nch; c += 32) {
        float v[16];
        tmem_ld16(cta.tmem + lane + c, v);
        if (!on || !drv.ok) continue;
        const int64_t o = (row0 + t) * O + n0 + c;
        if (j == 0) {
          float* dst = p.log_alpha + o;
#pragma unroll
          for (int q4 = 0; q4 < 16; q4 += 4)
            *reinterpret_cast<float4*>(dst + q4) = make_float4(gate_log_sigmoid(v[q4]), gate_log_sigmoid(v[q4 + 1]),
                                                               gate_log_sigmoid(v[q4 + 2]), gate_log_sigmoid(v[q4 + 3]));
        } else {
          float a8[8], b8[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) { a8[e] = gate_sigmoid(v[e]); b8[e] = gate_sigmoid(v[8 + e]); }
          T* dst = static_cast<T*>(p.out[j]) + o;
          Elt<T>::st8(dst, a8);
          Elt<T>::st8(dst + 8, b8);
        }
      }
    }
  }
  cta.finish();
}

}  // namespace muir
