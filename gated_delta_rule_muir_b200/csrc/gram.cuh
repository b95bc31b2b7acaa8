// The four decayed Grams of a unit (chunk of Cs <= 128 tokens of one (batch,
// head)):
//   M^kk_ts = k_t.Gam_{t<-s}.k_s,  M^ka_ts = k_t.Gam_{t<-s}.a_s        (s < t)
//   N^qk_ts = qt_t.Gam_{t<-s}.k_s, N^qa_ts = qt_t.Gam_{t<-s}.a_s       (s <= t)
// written as bf16 hi/lo images (sq_put layout) for the solve and map kernels.
//
// Boundary pivoting (openai-hub article, section "为 TPU 重写长序列并行算法";
// liuch.name post, bullet "Numerically-stable, large-chunk parallel kernel"):
// the unit's tokens form a binary tree of 8-token blocks. At level b (Cs/2, ...,
// 16, 8) the pivots are P = (2p+1) b, and every t in [P, P+b) meets every s in
// [P-b, P) with
//   Gam_{t<-s} = pre_t * suf_s,   pre_t = prod_{u=P..t} alpha_u,
//                                 suf_s = prod_{u=s+1..P-1} alpha_u,
// both products of alphas in [0, 1]. They are formed as 2^(sum of log2 alpha),
// a sum of non-positive terms: the running sum inside the token's 8-block plus
// the totals of the whole 8-blocks between it and the pivot. One tcgen05 product
// per level gives the blocks of all pivots at once:
//   XL rows p*2b + X*b + u = [K; Qt]_t * pre_t     (t = P + u, X = K, Qt)
//   YL rows p*2b + Y*b + u = [K; A]_s  * suf_s     (s = P - b + u, Y = K, A)
//   D = XL YL^T: row block p, column block p holds the pivot's four Gram blocks.
// Pairs inside one 8-token block (the 8x8 diagonal blocks) are computed exactly
// on the CUDA cores with running products of alphas while the tensor core
// works; the zeros right of the diagonal blocks are written by bulk stores.
//
// Staging: thread (g, J) owns channels 8g..8g+7 of 8-block J and walks its 8
// tokens in order (forward for an upper block, backward for a lower one), so the
// running sum stays in registers. The channel group varies fastest across the
// threads, so that a warp's load reads whole token rows (two rows of 256 bytes
// for dk = 128, not sixteen 32-byte pieces of sixteen rows), and XL and YL have
// 128-byte-swizzled rows (dk a multiple of 64), in which the 8 threads of a
// shared-memory phase, 8 consecutive channel groups of one row, store to 8
// distinct bank groups.
//
// TMEM: two 128-column slots, used by alternate levels; a level's results are
// drained while the next level's product runs. With bf16 inputs and one MMA pass
// the CTA needs about 106 KB of shared memory, so two units share an SM.
#pragma once

#include "chunk.cuh"

namespace muir {

// 8 floats as one bf16 row piece of a K-major tile: the hi plane, and with NS > 1 the lo plane too.
__device__ __forceinline__ uint32_t row_piece_off(const Tile& t, int m, int k8) {
  return (uint32_t)(m >> 3) * t.sbo + (uint32_t)(k8 >> 3) * 128u + (uint32_t)(m & 7) * 16u;
}
__device__ __forceinline__ uint32_t row_piece_off(const SwTile& t, int m, int k8) {
  return (uint32_t)(k8 >> 6) * t.box + (uint32_t)m * 128u + ((uint32_t)(((k8 >> 3) & 7) ^ (m & 7)) << 4);
}
template <int NS, typename OpTile>
__device__ __forceinline__ void put_row(const OpTile& t, int m, int k8, const float (&x)[8]) {
  if constexpr (NS == 1) {
    uint4 hi;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&hi);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
    sts128(t.hi + row_piece_off(t, m, k8), hi);
  } else {
    put_op(t, m, k8, x);
  }
}

constexpr float kLog2e = 1.4426950408889634f;

// 2^x for x <= 0 with the hardware's approximate base-2 exponential (relative
// error near 2^-22); results below the normal range flush to 0, the correct
// limit of a product of decays that underflows.
__device__ __forceinline__ float exp2_neg(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(fminf(x, 0.f)));
  return y;
}

template <int DK>
constexpr uint32_t gram_smem_bytes(int NS) {
  return 1024u                                      // alignment of the swizzled tiles
         + 2u * (NS > 1 ? 2u : 1u) * 128u * DK * 2u  // XL, YL: hi planes, and lo planes for NS > 1
         + 16u * DK * 4u                     // totals of the 8-blocks (log2)
         + 4u * 16u * DK * 4u                // rows of two diagonal blocks: k, qt, a, alpha
         + kZeroBuf;
}

template <int DK, typename T, int NS>
__global__ void __launch_bounds__(256, NS == 1 ? 2 : 1) gram_kernel(ChunkParams p) {
  extern __shared__ __align__(128) uint8_t sm[];
  __shared__ uint64_t bar;
  __shared__ uint32_t tslot;
  constexpr int G = DK / 8;
  constexpr uint32_t LB = 128u * DK * 2u;  // one bf16 plane of a 128-row operand tile
  constexpr uint32_t PL = NS > 1 ? 2u : 1u;  // planes per operand tile
  const int Cs = p.Cs, nb = Cs >> 3;
  const int nlev = Cs == 128 ? 4 : 3;  // b = Cs/2 .. 8
  const int lnb = Cs == 128 ? 4 : 3;   // log2(nb)
  const SubIdx s = sub_of(p, blockIdx.x, p.nsub, Cs);
  const int tid = threadIdx.x, warp = tid >> 5;
  const uint32_t base = (smem_u32(sm) + 1023u) & ~1023u;  // swizzled tiles start on 1024-byte boundaries
  uint8_t* const sma = sm + (base - smem_u32(sm));
  const auto XL = kmajor_tile<DK>(base, (PL - 1) * LB);
  const auto YL = kmajor_tile<DK>(base + PL * LB, (PL - 1) * LB);
  constexpr bool kSw = DK % 64 == 0;
  float* tot = reinterpret_cast<float*>(sma + 2 * PL * LB);  // [16][DK]
  float* drow = tot + 16 * DK;                               // [4][16][DK]
  const uint32_t zbuf = base + 2 * PL * LB + (16u * DK + 4u * 16u * DK) * 4u;
  uint8_t* out = p.gr + (int64_t)blockIdx.x * 4 * sq_bytes(Cs);
  const int64_t tok_stride = (int64_t)p.H * DK;
  const int64_t row0 = toff(p, s.b, s.tok0, s.h, DK);  // token 0 of the unit, channel 0

  if (Cs < 128) {  // rows >= Cs of the operands stay zero
    for (uint32_t pl = 0; pl < 2u * PL; ++pl) {
      if constexpr (kSw) {  // in every 64-column box of 128 rows
        for (uint32_t bx = 0; bx < DK / 64; ++bx)
          zero_smem(base + pl * LB + bx * 16384u + (uint32_t)Cs * 128u, (128u - Cs) * 128u);
      } else {
        zero_smem(base + pl * LB + (uint32_t)Cs * DK * 2u, (128u - Cs) * DK * 2u);
      }
    }
  }
  TcCta cta;
  cta.init(&tslot, &bar, 256);
  // zeros right of the diagonal 8-blocks of the four images, by the bulk-copy engine
  if (warp == 0) {
    const int lane = tid & 31;
    const uint32_t gb = (uint32_t)Cs * 16u;
    for (uint32_t o = lane * 16u; o < kZeroBuf; o += 512u) sts128(zbuf + o, make_uint4(0, 0, 0, 0));
    fence_async_smem();
    __syncwarp();
    for (int x = lane; x < 8 * nb; x += 32) {  // (image, hi/lo, row group)
      const int rg = x % nb, gh = x / nb;
      const uint32_t pb = (uint32_t)(rg + 1) * 128u;
      if (pb < gb) bulk_s2g(out + (gh >> 1) * sq_bytes(Cs) + (gh & 1) * sq_half(Cs) + rg * gb + pb, zbuf, gb - pb);
    }
    bulk_commit();
  }

  // ---- staging thread (g, J): channels 8g.., 8-block J --------------------
  const int sg = tid % G, sJ = tid / G;
  const bool stager = sJ < nb;
  const int c8 = sg * 8;
  if (stager) {
    // totals of the 8-block in log2 units
    float acc[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j] = 0.f;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      float la[8];
      ld8f(p.la + row0 + (int64_t)(8 * sJ + u) * tok_stride + c8, la);
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[j] = fmaf(la[j], kLog2e, acc[j]);
    }
    Elt<float>::st8(tot + sJ * DK + c8, acc);
  }
  __syncthreads();

  const T* kp = static_cast<const T*>(p.k);
  const T* qp = static_cast<const T*>(p.q);
  const T* ep = static_cast<const T*>(p.e);
  const T* gp = static_cast<const T*>(p.g);

  // Branch-free inside a warp: its lanes hold upper and lower blocks alike, so
  // the role (which rows, which walking direction, XL or YL) is selected per lane.
  auto stage = [&](int lev) {
    if (!stager) return;
    const int lb3 = lnb - 1 - lev;  // log2(b / 8)
    const int b = 8 << lb3;
    const bool upper = (sJ >> lb3) & 1;
    const int pv = sJ >> (lb3 + 1);
    const int P = (2 * pv + 1) * b, JP = P >> 3;
    // whole 8-blocks between this block and the pivot
    float off[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) off[j] = 0.f;
    const int j0 = upper ? JP : sJ + 1, j1 = upper ? sJ : JP;
    for (int jb = j0; jb < j1; ++jb) {
      float tb[8];
      lds_vec(tot + jb * DK + c8, tb);
#pragma unroll
      for (int j = 0; j < 8; ++j) off[j] += tb[j];
    }
    const int lo = upper ? P : P - b;  // first token of the half
    const int rbase = pv * 2 * b;
    const T* x1p = upper ? qp : ep;                  // q (then r g q) or e (then e k)
    const T* x2p = upper && gp ? gp : kp;            // g, or a stand-in that is not used
    const bool use_g = upper && gp != nullptr;
    const auto dst = upper ? XL : YL;
    float rl[8];  // r of these channels (loaded here: an array captured by the lambda would live in local memory)
    ld8f(p.r + (int64_t)s.h * DK + c8, rl);
    float run[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) run[j] = 0.f;
    constexpr int BT = NS == 1 ? 2 : (sizeof(T) == 2 ? 8 : 4);  // tokens per load batch
#pragma unroll 1
    for (int u0 = 0; u0 < 8; u0 += BT) {
      Pack8<T> pk[BT], p1[BT], p2[BT];
      Pack8<float> pl[BT];
#pragma unroll
      for (int v = 0; v < BT; ++v) {
        const int w8 = upper ? u0 + v : 7 - (u0 + v);  // offset of the token in its block
        const int64_t o = row0 + (int64_t)(8 * sJ + w8) * tok_stride + c8;
        pk[v].ld(kp + o);
        pl[v].ld(p.la + o);
        p1[v].ld(x1p + o);
        p2[v].ld(x2p + o);
      }
#pragma unroll
      for (int v = 0; v < BT; ++v) {
        const int w8 = upper ? u0 + v : 7 - (u0 + v);
        float kk[8], x1[8], x2[8], la[8];
        pk[v].get(kk);
        p1[v].get(x1);
        p2[v].get(x2);
        pl[v].get(la);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float l2 = la[j] * kLog2e;
          // pre_t includes alpha_t (upper); suf_s covers the alphas after s (lower)
          const float f = exp2_neg(run[j] + (upper ? l2 : 0.f) + off[j]);
          run[j] += l2;
          const float m1 = upper ? rl[j] * (use_g ? x2[j] : 1.f) : kk[j];  // r g, or k
          x1[j] = x1[j] * m1 * f;
          kk[j] *= f;
        }
        const int uu = 8 * sJ + w8 - lo, q8 = uu >> 3;
        const int m = rbase + 8 * q8 + w8;
        put_row<NS>(dst, m, c8, kk);
        put_row<NS>(dst, m + b, c8, x1);
      }
    }
  };

  // ---- epilogue of one level: TMEM slot -> the four images ----------------
  const int rho = tid & 127, wg = tid >> 7;
  auto drain = [&](int lev) {
    const int lb3 = lnb - 1 - lev, b = 8 << lb3;
    const uint32_t col0 = (uint32_t)(lev & 1) * 128u;
    const uint32_t lane_addr = cta.tmem + tmem_lane_base(warp) + col0;
    const int pv = rho / (2 * b);
    const int X = (rho / b) & 1, within = rho % b;
    const int P = (2 * pv + 1) * b;
    const int t = P + within;
    const bool on = rho < Cs;
    // this warpgroup's columns of the row's pivot: Y = wg, [pv*2b + wg*b, + b)
    for (int cq = 0; cq < b; cq += 8) {
      float v[8];
      if (b >= 16) {  // the warp's 32 rows share one pivot: warp-uniform columns
        tmem_ld8(lane_addr + (uint32_t)(pv * 2 * b + wg * b + cq), v);
      } else {        // b = 8: the warp spans two pivots; load both and keep this row's
        const int pw = ((warp & 3) * 32) / (2 * b);
        float v0[8], v1[8];
        tmem_ld8(lane_addr + (uint32_t)(pw * 2 * b + wg * b), v0);
        tmem_ld8(lane_addr + (uint32_t)((pw + 1) * 2 * b + wg * b), v1);
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = pv == pw ? v0[j] : v1[j];
      }
      if (on) sq_put(out + (2 * X + wg) * sq_bytes(Cs), Cs, t, P - b + cq, v);
    }
  };

  // ---- the 8x8 diagonal blocks, two per step, on the CUDA cores -----------
  // warp w takes row w of block J (w + 1 pairs) and row 7 - w of block J + 1
  // (8 - w pairs): 9 pairs for every warp. Thread (row t, lane ln of 32) holds
  // CD = DK/32 channels; for s = t, t-1, ... the running product
  // Gam_{t<-s} = Gam_{t<-s+1} alpha_{s+1} scales both right operands; the 32
  // partial sums (4 Grams x 8 columns) are reduced over the 32 lanes of the row,
  // after which lane ln holds Gram ln/8, column ln%8.
  Pack8<T> fk, fe, fq, fg;
  Pack8<float> fl;
  auto fetch = [&](int J, int nblk) {  // rows of blocks J .. J + nblk - 1, one piece per thread
    if (tid < nblk * 8 * G) {
      const int tok = tid / G, cg = tid % G;
      const int64_t o = row0 + (int64_t)(8 * J + tok) * tok_stride + 8 * cg;
      fk.ld(kp + o);
      fe.ld(ep + o);
      fq.ld(qp + o);
      fg.ld_or_one(gp ? gp + o : nullptr);
      fl.ld(p.la + o);
    }
  };
  auto put_rows = [&](int nblk) {
    if (tid < nblk * 8 * G) {
      const int tok = tid / G, cg = tid % G;
      float kk[8], ee[8], qq[8], gg[8], la[8], rr[8];
      fk.get(kk);
      fe.get(ee);
      fq.get(qq);
      fg.get(gg);
      fl.get(la);
      ld8f(p.r + (int64_t)s.h * DK + 8 * cg, rr);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        la[j] = exp2_neg(la[j] * kLog2e);
        ee[j] *= kk[j];
        qq[j] = rr[j] * gg[j] * qq[j];
      }
      float* d0 = drow + tok * DK + 8 * cg;
      Elt<float>::st8(d0 + 0 * 16 * DK, kk);
      Elt<float>::st8(d0 + 1 * 16 * DK, qq);
      Elt<float>::st8(d0 + 2 * 16 * DK, ee);
      Elt<float>::st8(d0 + 3 * 16 * DK, la);
    }
  };
  constexpr int CD = DK / 32;  // channels per lane in the diagonal blocks
  // row t of block J, whose rows sit at drow tokens 8 blk ..
  auto diag_row = [&](int J, int blk, int t) {
    const int ln = tid & 31, c0 = ln * CD;
    const float* dr = drow + blk * 8 * DK;
    float xk[CD], xq[CD], gm[CD];
    lds_vec(dr + 0 * 16 * DK + t * DK + c0, xk);
    lds_vec(dr + 1 * 16 * DK + t * DK + c0, xq);
#pragma unroll
    for (int j = 0; j < CD; ++j) gm[j] = 1.f;
    float v[32];
#pragma unroll
    for (int ss = 7; ss >= 0; --ss) {
      float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
      if (ss <= t) {
        float yk[CD], ya[CD], al[CD];
        lds_vec(dr + 0 * 16 * DK + ss * DK + c0, yk);
        lds_vec(dr + 2 * 16 * DK + ss * DK + c0, ya);
        lds_vec(dr + 3 * 16 * DK + ss * DK + c0, al);
#pragma unroll
        for (int j = 0; j < CD; ++j) {
          yk[j] *= gm[j];
          ya[j] *= gm[j];
          a0 += xk[j] * yk[j]; a1 += xk[j] * ya[j]; a2 += xq[j] * yk[j]; a3 += xq[j] * ya[j];
          gm[j] *= al[j];
        }
      }
      v[0 * 8 + ss] = a0; v[1 * 8 + ss] = a1; v[2 * 8 + ss] = a2; v[3 * 8 + ss] = a3;
    }
#pragma unroll
    for (int m = 16, n = 16; m >= 1; m >>= 1, n >>= 1) {
      const bool up = (ln & m) != 0;
#pragma unroll
      for (int j = 0; j < n; ++j) {
        const float send = up ? v[j] : v[j + n];
        const float keep = up ? v[j + n] : v[j];
        v[j] = keep + __shfl_xor_sync(0xffffffffu, send, m);
      }
    }
    const int g = ln >> 3, ss = ln & 7;
    const bool keep = ss < t || (g >= 2 && ss == t);  // M^kk, M^ka exclude the diagonal
    const float w = keep ? v[0] : 0.f;
    const __nv_bfloat16 hb = __float2bfloat16_rn(w);
    const __nv_bfloat16 lb = __float2bfloat16_rn(w - __bfloat162float(hb));
    const int r = 8 * J + t, c = 8 * J + ss;
    const uint32_t o = (uint32_t)(r >> 3) * (uint32_t)Cs * 16u + (uint32_t)(c >> 3) * 128u + (uint32_t)(r & 7) * 16u +
                       (uint32_t)(c & 7) * 2u;
    uint8_t* img = out + g * sq_bytes(Cs);
    *reinterpret_cast<__nv_bfloat16*>(img + o) = hb;
    *reinterpret_cast<__nv_bfloat16*>(img + sq_half(Cs) + o) = lb;
  };
  // blocks J (.. J + 1 when nblk = 2); their rows were fetched before, those of
  // the next step (nnext blocks from `next`, if any) are fetched here, under this
  // step's arithmetic
  auto diag_step = [&](int J, int nblk, int next, int nnext) {
    __syncthreads();  // drow is free
    put_rows(nblk);
    __syncthreads();
    if (next >= 0) fetch(next, nnext);
    const int w = tid >> 5;
    diag_row(J, 0, w);
    if (nblk == 2) diag_row(J + 1, 1, 7 - w);
  };

  const uint32_t id = idesc_bf16(128, Cs, 0, 0);
  uint32_t phase = 0;
  bool ok = true;
  int it = 0;
  for (int lev = 0; lev < nlev; ++lev) {
    stage(lev);
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      mma_ops(cta.tmem + (uint32_t)(lev & 1) * 128u, kview(XL), kview(YL), DK / 16, id, NS, false);
      mma_commit(&bar);
    }
    // the diagonal-block rows are fetched level by level, so that no prefetched
    // registers stay live across the staging
    const int it1 = (lev + 1) * nb / nlev;
    if (it < it1) fetch(it, it1 - it < 2 ? it1 - it : 2);
    if (lev > 0) drain(lev - 1);  // the other slot, complete since the last wait
    while (it < it1) {
      const int nblk = it1 - it < 2 ? it1 - it : 2, nx = it + nblk;
      diag_step(it, nblk, nx < it1 ? nx : -1, it1 - nx < 2 ? it1 - nx : 2);
      it = nx;
    }
    ok = __syncthreads_and(tid == 0 ? (mbar_wait(&bar, phase) ? 1 : 0) : 1) != 0;  // one poller
    phase ^= 1u;
    tc_fence_after();
    if (!ok) break;  // no further product is issued; the kernel winds down
  }
  if (ok) drain(nlev - 1);
  if (warp == 0) bulk_wait_all();  // the zero stores have read their source
  cta.finish();
}

}  // namespace muir
