// Chunkwise backward pass (reverse mode of the chunk map in chunk.cuh).
//
// Per unit (chunk of Cs <= 128 tokens) with start state S0, forward quantities
//   Z = (K*Gam) S0 + M^kk U,  P = T Z,  O = (Qt*Gam) S0 + N^qk U - N^qa P,
//   S_C = Diag(Gam_C) S0 + (K*Gsuf)^T U - (A*Gsuf)^T P,  y = z*O,
// and cotangents dO = z*dy, dS_C (state cotangent at the unit end):
//   dP   = -N^qa^T dO - (A*Gsuf) dS_C          dZ = T^T dP
//   dU   = N^qk^T dO + (K*Gsuf) dS_C + M^kk^T dZ
//   dQp  = dO S0^T      dKp = dZ S0^T      dKs = U dS_C^T      dAs = -P dS_C^T
//   dN^qk = dO U^T, dN^qa = -dO P^T (s <= t);  dM^kk = dZ U^T, dM^ka = -dZ P^T (s < t)
//   dGam_C = rowsum(dS_C * S0)
// (dM^ka uses d(T) = -T d(M^ka) T, so -T^T dP Z^T T^T = -dZ P^T.) The state
// cotangent entering the unit is the adjoint of the unit's affine map:
//   dS0 = Phi^T dS_C + Q'^T dO.
// A decayed Gram G_ts = sum_i X_ti Y_si Gam_{t<-s,i} sends
//   dX_t = sum_s dG_ts Y_s*Gam_{t<-s},  dY_s = sum_t dG_ts X_t*Gam_{t<-s},
// and, since Gam_{t<-s} = exp(L_t - L_s) with L the in-chunk cumulative sum of
// log alpha, dL_t += X_t*dX_t and dL_s -= Y_s*dY_s. dlog_alpha is the reverse
// cumulative sum of dL inside the unit.
//
// Kernels:
//   bwd_pe_kernel      P = W S0 + Ut, dz = dy * (Q' S0 + Oloc), E = Q'^T dO
//   rscan_kernel       reverse sweep over units per (b, h, kSlab-column slab):
//                      dS <- Phi^T dS + E (the adjoint of the state map)
//   bwd_dz_kernel      dP, dZ, dU (written as dv = w dU, dw = v dU)
//   bwd_grads_kernel   dQp, dKp, dKs, dAs, dGam_C and the four Gram cotangents
//   bwd_gram_kernel    the Gram backward: tree levels on tcgen05 (left and
//                      right phases), exact diagonal blocks on the CUDA cores
//   bwd_final_kernel   decay cotangents, reverse cumsum, chain rule to inputs
#pragma once

#include "chunk.cuh"

namespace muir {

struct BwdBufs {
  float* S_chunks;  // [nst][dk][dv]
  float* dSC;       // [nst][dk][dv]   state cotangent at each unit's end
  float* P;         // [nst][Cs][dv]
  float* dZ;        // [nst][Cs][dv]
  float* eC;        // [nst][dk]: rowsum(dS_C * S_C), all that lands on the unit's last log-decay
  float* E;         // [nst][dv/kSlab][dk][kSlab]: Q'^T dO per unit, column slabs (slab_off)
  float* g4;        // [nst][4][Cs][dk]: dQp, dKp, dKs, dAs
  float* dG;        // [nst][4][Cs][Cs]: dM^kk, dM^ka, dN^qk, dN^qa
  float* gl;        // [nst][4][Cs][dk]: dK_left, dQ_left, dK_right, dA_right
  const float* dS_T;
  float* dS0;
  void *dq, *dk, *dv, *de, *dw, *dg;
  float* dla;
  float* dr;
};

// ---------------------------------------------------------------------------
// rscan_kernel: the sequential part of the backward pass. For n = last..0:
//   dSC[n] = dS;   dS <- Phi_n^T dS + E_n,   E_n = Q'_n^T dO_n (from bwd_pe)
// A = Phi^T: tile 0 of the map image read through the transposed view; B = dS
// (K = key row, N = kSlab slab columns, MN-major) from registers. Phi_n and the
// E_n slab arrive by bulk copies into two alternating buffers, two units ahead.
// ---------------------------------------------------------------------------
template <int DK, int NS>
__global__ void __launch_bounds__(128, 1) rscan_kernel(ChunkParams p, BwdBufs q) {
  extern __shared__ __align__(128) uint8_t sm[];
  __shared__ uint64_t bar, bar_c[2];
  __shared__ uint32_t tslot;
  constexpr int NW = kSlab;
  const int dv = p.dv, slabs = dv / NW;
  const int slab = blockIdx.x % slabs;
  const int bh = blockIdx.x / slabs;
  const int h = bh % p.H, b = bh / p.H;
  const int tid = threadIdx.x, warp = tid >> 5;
  const MapGeom g = map_geom(DK, p.Cs);
  const uint32_t ES = DK * NW * 4u;
  const uint32_t base = smem_u32(sm);
  const uint32_t e_off = 2 * g.tile;  // the transposed view may read up to 2 KB past a Phi tile: E follows
  const uint32_t b_off = e_off + 2 * ES;
  const Tile Bt{base + b_off, base + b_off + NW * DK * 2u, 128u, DK * 16u};
  if (tid == 0) {
    mbar_init(&bar_c[0], 1);
    mbar_init(&bar_c[1], 1);
  }
  TcCta cta;
  cta.init(&tslot, &bar, 32);
  MmaSync drv{&bar, 0u, true};
  const uint32_t lane = tmem_lane_base(warp);
  const float* e_s = reinterpret_cast<const float*>(static_cast<const uint8_t*>(sm) + e_off);
  auto uid_of = [&](int n) { return ((int64_t)b * p.H + h) * p.nsub + n; };
  auto issue = [&](int n, int buf) {
    if (tid == 0) {
      mbar_expect_tx(&bar_c[buf], g.tile + ES);
      bulk_g2s_big(base + buf * g.tile, p.ma + uid_of(n) * g.unit, g.tile, &bar_c[buf]);
      bulk_g2s_big(base + e_off + buf * ES, reinterpret_cast<const uint8_t*>(q.E + (uid_of(n) * slabs + slab) * DK * NW),
                   ES, &bar_c[buf]);
    }
  };
  float ds[NW];
  {
    const float* src = q.dS_T ? q.dS_T + (((int64_t)b * p.H + h) * DK) * dv + slab * NW : nullptr;
#pragma unroll
    for (int j = 0; j < NW; ++j) ds[j] = (src && tid < DK) ? src[(int64_t)tid * dv + j] : 0.f;
  }
  const uint32_t id = idesc_bf16(128, NW, 1, 1);
  issue(p.nsub - 1, 0);
  if (p.nsub > 1) issue(p.nsub - 2, 1);
  for (int k = 0; k < p.nsub && drv.ok; ++k) {
    const int n = p.nsub - 1 - k;
    const int buf = k & 1;
    if (tid < DK) {
#pragma unroll
      for (int j = 0; j < NW; j += 8) {
        float v[8];
#pragma unroll
        for (int e2 = 0; e2 < 8; ++e2) v[e2] = ds[j + e2];
        put_mn(Bt, tid, j, v);
      }
    }
    fence_async_smem();  // the cotangent operand is visible to the tensor core after the barrier below
    tc_fence_before();
    const bool c_ok = mbar_wait(&bar_c[buf], (uint32_t)(k >> 1) & 1u);
    if (!__syncthreads_and(c_ok ? 1 : 0)) { drv.ok = false; break; }
    const Tile PhiT{base + buf * g.tile, base + buf * g.tile + g.half, DK * 16u, 128u};
    drv.run_synced([&] { mma_tiles(cta.tmem, PhiT, Bt, DK / 16, id, NS, false); },
                    [&] {  // the unit's state cotangent leaves while the tensor core works
                      if (tid < DK) {
                        float* o = q.dSC + (uid_of(n) * DK + tid) * dv + slab * NW;
#pragma unroll
                        for (int j = 0; j < NW; j += 8) stg256(o + j, *reinterpret_cast<const float(*)[8]>(&ds[j]));
                      }
                    });
    if (!drv.ok) break;
    float v[NW];
    tmem_ld_slab(cta.tmem + lane, v);
    if (tid < DK) {
      const float* add = e_s + buf * (ES / 4) + tid * NW;
#pragma unroll
      for (int j = 0; j < NW; j += 4) {
        const float4 a4 = *reinterpret_cast<const float4*>(add + j);
        ds[j] = v[j] + a4.x; ds[j + 1] = v[j + 1] + a4.y; ds[j + 2] = v[j + 2] + a4.z; ds[j + 3] = v[j + 3] + a4.w;
      }
    }
    __syncthreads();
    if (k + 2 < p.nsub) issue(n - 2, buf);
  }
  if (q.dS0 && tid < DK && drv.ok) {
    float* o = q.dS0 + (((int64_t)b * p.H + h) * DK + tid) * dv + slab * NW;
#pragma unroll
    for (int j = 0; j < NW; j += 8) stg256(o + j, *reinterpret_cast<const float(*)[8]>(&ds[j]));
  }
  cta.finish();
}

// Stage a row-major fp32 matrix src[rows][cols] (row stride ld) as an MN-major
// operand contracting over rows (put_mn), values scaled by sign. rows <= 128 and
// a multiple of 8, cols / 8 a power of two.
__device__ __forceinline__ void stage_rows_mn(const Tile& t, const float* src, int rows, int cols, int64_t ld,
                                              float sign) {
  #pragma unroll 4
  for (int x = threadIdx.x; x < rows * (cols / 8); x += blockDim.x) {
    int r, c8;
    piece_of_rt(x, cols / 8, r, c8);
    float v[8];
    ld8f(src + r * ld + c8, v);
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] *= sign;
    put_mn(t, r, c8, v);
  }
}

// ---------------------------------------------------------------------------
// bwd_pe_kernel (per unit, after the recompute sweep):
//   P  = W S0 + Ut                  A = W (K-major over key channels), B = S0
//   dz = dy * (Q' S0 + Oloc)        A = Q' (tile 1 of the map image, bulk copy)
//   E  = Q'^T dO,  dO = z * dy      A = Q' through the transposed view, B = dO
// TMEM: P -> 0, O -> 128, E -> 256.
// ---------------------------------------------------------------------------
template <int DK, int DV, typename T, int NS>
__global__ void __launch_bounds__(256, 1) bwd_pe_kernel(ChunkParams p, BwdBufs q) {
  extern __shared__ __align__(128) uint8_t sm[];
  __shared__ uint64_t bar, bar_cp, bar_s;
  __shared__ uint32_t tslot;
  const int Cs = p.Cs;
  const SubIdx s = sub_of(p, blockIdx.x, p.nsub, Cs);
  constexpr int NT = 256;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int64_t u = blockIdx.x;
  const MapGeom g = map_geom(DK, Cs);
  const uint32_t base = smem_u32(sm);
  constexpr uint32_t TB = 128u * 128u * 2u;
  const Tile Qt{base, base + g.half, 128u, DK * 16u};        // Q': rows = tokens, K = key channel
  const Tile QtT{base, base + g.half, DK * 16u, 128u};       // Q'^T: M = key channel, K = token
  const Tile A{base + 2 * TB, base + 3 * TB, 128u, DK * 16u};  // W: rows = tokens, K = key channel
  const Tile B{base + 4 * TB, base + 5 * TB, 128u, DK * 16u};  // S0: K = key channel, N = value column
  // dO: K = token, N = value column, staged by a row-major sweep; a 16-byte pad
  // between the 8-column blocks keeps the stores of a shared-memory phase in 8
  // distinct bank groups
  const Tile Bo{base + 4 * TB, base + 5 * TB + 256u, 128u, (uint32_t)Cs * 16u + 16u};
  if (tid == 0) {
    mbar_init(&bar_cp, 1);
    mbar_init(&bar_s, 1);
  }
  TcCta cta;
  cta.init(&tslot, &bar, 512);
  if (tid == 0) {
    mbar_expect_tx(&bar_cp, g.tile);
    bulk_g2s_big(base, p.ma + u * g.unit + g.tile, g.tile, &bar_cp);
  }
  MmaSync drv{&bar, 0u, true};
  const uint32_t lane = tmem_lane_base(warp);
  const float* S0 = q.S_chunks + u * DK * DV;
  uint32_t ph_s = 0;
  bool st_ok = stage_raw<false>(A, p.wsave + u * Cs * DK, Cs, DK, 1.f, &bar_s, ph_s);
  st_ok = stage_raw<true>(B, S0, DK, DV, 1.f, &bar_s, ph_s) && st_ok;
  drv.ok = __syncthreads_and((mbar_wait(&bar_cp, 0) && st_ok) ? 1 : 0) != 0;
  const uint32_t id = idesc_bf16(128, DV, 0, 1);
  if (drv.ok)
    drv.run([&] {
      mma_tiles(cta.tmem + 0, A, B, DK / 16, id, NS, false);
      mma_tiles(cta.tmem + 128, Qt, B, DK / 16, id, NS, false);
    });
  const int t = tid & 127, wg = tid >> 7;  // TMEM row; warpgroups split the columns
  // dO = z * dy (B region is free: both MMAs above have completed)
  stage_prod<T, true, DV>(Bo, p, s, Cs, static_cast<const T*>(p.dy), static_cast<const T*>(p.z), nullptr, 1.f);
  if (drv.ok) drv.run([&] { mma_tiles(cta.tmem + 256, QtT, Bo, Cs / 16, idesc_bf16(128, DV, 1, 1), NS, false); });
  const float* Ut = p.usave + u * Cs * DV;
  const float* olu = p.ol + u * Cs * DV;
  float* P = q.P + u * Cs * DV;
  {
    // P = W S0 + Ut and dz = dy * (Q' S0 + Oloc) by 32 x 32 row blocks (rows_fill,
    // rows_store): Ut, Oloc and dy come in and P, dz go out in whole lines. All
    // shared memory is free here, the MMAs having completed.
    const int ln = tid & 31, row0 = 32 * (warp & 3);
    const bool wdz = p.dz && p.z;
    const int64_t ts = (int64_t)p.H * DV;
    const int64_t o0 = toff(p, s.b, s.tok0, s.h, DV);
    constexpr uint32_t FB = row_block_bytes<float>(), CB = 2 * FB + row_block_bytes<T>();  // Ut, Oloc, dy blocks
    constexpr int NCK = (DV + 63) / 64;  // 32-column chunks per warp
    static_assert(8u * NCK * CB <= 6u * 128u * 128u * 2u, "row blocks exceed the tiles' shared memory");
    const uint32_t wb = base + (uint32_t)warp * NCK * CB;
    uint8_t* const wsm = sm + (wb - base);
    if (drv.ok) {
      int k = 0;
      for (int c = wg * 32; c < DV; c += 64, ++k) {
        rows_fill<float>(wb + k * CB, Ut, DV, row0, Cs, c);
        if (wdz) {
          rows_fill<float>(wb + k * CB + FB, olu, DV, row0, Cs, c);
          rows_fill<T>(wb + k * CB + 2 * FB, static_cast<const T*>(p.dy) + o0, ts, row0, Cs, c);
        }
      }
    }
    cp_async_wait_all();
    __syncwarp();
    {
      int k = 0;
      for (int c = wg * 32; c < DV; c += 64, ++k) {
        uint8_t* bu = wsm + k * CB;
        float v[32];
        tmem_ld32(cta.tmem + lane + c, v);
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8) {
          float a8[8];
          row8_get<float>(bu, ln, q8, a8);
#pragma unroll
          for (int j = 0; j < 8; ++j) a8[j] += v[8 * q8 + j];
          row8_put(bu, ln, q8, a8);
        }
        if (wdz) {
          tmem_ld32(cta.tmem + lane + 128 + c, v);
#pragma unroll
          for (int q8 = 0; q8 < 4; ++q8) {
            float ol8[8], dd[8];
            row8_get<float>(bu + FB, ln, q8, ol8);
            row8_get<T>(bu + 2 * FB, ln, q8, dd);
#pragma unroll
            for (int j = 0; j < 8; ++j) ol8[j] = dd[j] * (v[8 * q8 + j] + ol8[j]);
            row8_put(bu + FB, ln, q8, ol8);
          }
        }
      }
    }
    __syncwarp();
    if (drv.ok) {
      int k = 0;
      for (int c = wg * 32; c < DV; c += 64, ++k) {
        rows_store<float>(wsm + k * CB, P, DV, row0, Cs, c);
        if (wdz) rows_store<T>(wsm + k * CB + FB, static_cast<T*>(p.dz) + o0, ts, row0, Cs, c);
      }
    }
  }
  float* E = q.E + u * DK * DV;
  for (int c = wg * 16; c < DV; c += 32) {
    float v[16];
    tmem_ld16(cta.tmem + lane + 256 + c, v);
    if (t < DK && drv.ok) {
      float* o = E + slab_off(c, t, DK);
      stg_row16(o, v);
    }
  }
  cta.finish();
}

// ---------------------------------------------------------------------------
// bwd_dz_kernel: dP = -N^qa^T dO - (A*Gsuf) dS_C;  dZ = T^T dP;
//                dU = N^qk^T dO + (K*Gsuf) dS_C + M^kk^T dZ.
// TMEM: dP -> 0, dU -> 128, dZ -> 256. Tiles: A, B1 (dO), B2 (dS_C; later dZ).
// ---------------------------------------------------------------------------
template <int DK, int DV, typename T, int NS>
__global__ void __launch_bounds__(256, 1) bwd_dz_kernel(ChunkParams p, BwdBufs q) {
  extern __shared__ __align__(128) uint8_t sm[];
  __shared__ uint64_t bar, bar_cp;
  __shared__ uint32_t tslot;
  const int Cs = p.Cs;
  const SubIdx s = sub_of(p, blockIdx.x, p.nsub, Cs);
  constexpr int NT = 256;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int64_t u = blockIdx.x;
  const uint32_t base = (smem_u32(sm) + 1023u) & ~1023u;  // swizzled tiles start on 1024-byte boundaries
  constexpr uint32_t TB = 128u * 128u * 2u, TBP = TB + 256u;
  const uint32_t ks = (uint32_t)Cs * 16u;
  const uint32_t H = sq_half(Cs);
  const Tile AT{base, base + H, ks, 128u};      // transposed view of a Gram / T image: M = column, K = row
  const auto Ak = kmajor_tile<DK>(base, TB);  // staged operand over channels (K = DK), row-major sweep
  // dO, staged by a row-major sweep as an MN-major tile: a 16-byte pad between
  // the 8-column blocks puts the 8 stores of a shared-memory phase (8
  // consecutive column blocks of one token row) in 8 distinct bank groups
  const Tile B1{base + 2 * TB, base + 2 * TB + TBP, 128u, ks + 16u};
  const uint32_t b2 = base + 2 * TB + 2 * TBP;
  const Tile B2{b2, b2 + TB, 128u, DK * 16u};
  const Tile B3{b2, b2 + TB, 128u, ks};
  if (tid == 0) mbar_init(&bar_cp, 1);
  zero_smem(base + 2 * TB, 2 * TBP + 2 * TB);
  TcCta cta;
  cta.init(&tslot, &bar, 512);
  MmaSync drv{&bar, 0u, true};
  const uint32_t lane = tmem_lane_base(warp);
  const uint8_t* G = p.gr + u * 4 * sq_bytes(Cs);
  const float* gsuf = p.dec + (u * 4 + 3) * Cs * DK;
  const int t = tid & 127, wg = tid >> 7;  // TMEM row; warpgroups split the columns
  constexpr uint32_t cP = 0, cU = 128, cZ = 256;
  uint32_t cp_phase = 0;
  // image copies into the A region: issue_img starts one (no MMA may be reading
  // the region), wait_img waits for it; work that does not touch A runs between
  auto issue_img = [&](const uint8_t* img) {
    if (tid == 0) {
      mbar_expect_tx(&bar_cp, 2 * H);
      bulk_g2s_big(base, img, 2 * H, &bar_cp);
    }
  };
  auto wait_img = [&] {
    const bool ok = mbar_wait(&bar_cp, cp_phase);
    cp_phase ^= 1u;
    if (!ok) drv.ok = false;
  };
  auto load_img = [&](const uint8_t* img) {
    issue_img(img);
    wait_img();
  };
  issue_img(G + 3 * sq_bytes(Cs));  // N^qa -> -dP (partial): N^qa^T dO
  // B1 = dO = z * dy (K = token, N = value column)
  stage_prod<T, true, DV>(B1, p, s, Cs, static_cast<const T*>(p.dy), static_cast<const T*>(p.z), nullptr, 1.f);
  stage_rows_mn(B2, q.dSC + u * DK * DV, DK, DV, DV, 1.f);  // dS_C (K = channel)
  const uint32_t idT = idesc_bf16(128, DV, 1, 1), idK = idesc_bf16(128, DV, 0, 1);
  wait_img();
  drv.run([&] { mma_tiles(cta.tmem + cP, AT, B1, Cs / 16, idT, NS, false); });
  load_img(G + 2 * sq_bytes(Cs));  // N^qk -> dU: N^qk^T dO
  drv.run([&] { mma_tiles(cta.tmem + cU, AT, B1, Cs / 16, idT, NS, false); });
  // (A*Gsuf) and (K*Gsuf): rows s, K = channel (K-major)
  auto stage_suf = [&](bool erase) {
    stage_prod<T, false, DK>(Ak, p, s, Cs, static_cast<const T*>(p.k), erase ? static_cast<const T*>(p.e) : nullptr,
                             gsuf, 1.f);
  };
  stage_suf(true);
  drv.run([&] { mma_ops(cta.tmem + cP, kview(Ak), NoSw{B2}, DK / 16, idK, NS, true); });  // -dP = N^qa^T dO + (A*Gsuf) dS_C
  stage_suf(false);
  drv.run([&] { mma_ops(cta.tmem + cU, kview(Ak), NoSw{B2}, DK / 16, idK, NS, true); });  // + (K*Gsuf) dS_C
  // dP (TMEM, negated) -> B3 (K = token), then dZ = T^T dP
  issue_img(p.tt + u * sq_bytes(Cs));  // T^T
  for (int c = wg * 16; c < DV; c += 32) {
    float v[16];
    tmem_ld16(cta.tmem + lane + cP + c, v);
    if (t < Cs) {
      float a8[8], b8[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) { a8[j] = -v[j]; b8[j] = -v[8 + j]; }
      put_mn(B3, t, c, a8);
      put_mn(B3, t, c + 8, b8);
    }
  }
  wait_img();
  drv.run([&] { mma_tiles(cta.tmem + cZ, AT, B3, Cs / 16, idT, NS, false); });
  float* dZo = q.dZ + u * Cs * DV;
  issue_img(G + 0 * sq_bytes(Cs));  // M^kk^T (A is free: the T^T product has completed)
  for (int c = wg * 16; c < DV; c += 32) {
    float v[16];
    tmem_ld16(cta.tmem + lane + cZ + c, v);
    if (t < Cs) {
      float a8[8], b8[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) { a8[j] = v[j]; b8[j] = v[8 + j]; }
      put_mn(B3, t, c, a8);
      put_mn(B3, t, c + 8, b8);
    }
  }
  // dZ out in whole lines through dO's memory (free since its two products)
  drain_rows(cta.tmem + lane, cZ, DV, dZo, DV, Cs, reinterpret_cast<float*>(sm + (base + 2 * TB - smem_u32(sm))),
             drv.ok, [](int, int, float(&)[32]) {});
  wait_img();
  // dU -> dv = w dU and dw = v dU by 32 x 32 row blocks (rows_fill, rows_store):
  // w and v come in whole lines, into dO's tile (free since its two products)
  // while the last product runs where they fit there, and dv, dw go out through
  // the A tile's memory once that product has completed.
  constexpr uint32_t IB = row_block_bytes<T>(), OB = row_block_bytes<float>();
  constexpr int NCK = (DV + 63) / 64;  // 32-column chunks per warp
  constexpr bool kFillUnder = 8u * NCK * 2u * IB <= 2u * TBP;
  static_assert(8u * 2u * OB <= 2u * TB, "output row blocks exceed the A tile");
  static_assert(8u * NCK * 2u * IB <= 2u * TB + 2u * TBP, "input row blocks exceed the free tiles");
  const int ln = tid & 31, row0 = 32 * (warp & 3);
  const int64_t ts = (int64_t)p.H * DV, o0 = toff(p, s.b, s.tok0, s.h, DV);
  const uint32_t inb = base + 2 * TB + (uint32_t)warp * NCK * 2u * IB;  // after the A tile
  const uint32_t outb = base + (uint32_t)warp * 2u * OB;
  auto gen = [&](uint32_t x) { return sm + (x - smem_u32(sm)); };  // shared address -> generic pointer
  auto fill = [&] {
    if (drv.ok) {
      int k = 0;
      for (int c = wg * 32; c < DV; c += 64, ++k) {
        rows_fill<T>(inb + 2u * k * IB, static_cast<const T*>(p.w) + o0, ts, row0, Cs, c);
        rows_fill<T>(inb + (2u * k + 1u) * IB, static_cast<const T*>(p.v) + o0, ts, row0, Cs, c);
      }
    }
    cp_async_wait_all();
  };
  drv.run_overlap([&] { mma_tiles(cta.tmem + cU, AT, B3, Cs / 16, idT, NS, true); },
                  [&] {
                    if constexpr (kFillUnder) fill();
                  });
  if constexpr (!kFillUnder) fill();
  __syncwarp();
  {
    int k = 0;
    for (int c = wg * 32; c < DV; c += 64, ++k) {
      float v[32];
      tmem_ld32(cta.tmem + lane + cU + c, v);
#pragma unroll
      for (int q8 = 0; q8 < 4; ++q8) {
        float ww[8], vv[8];
        row8_get<T>(gen(inb + 2u * k * IB), ln, q8, ww);
        row8_get<T>(gen(inb + (2u * k + 1u) * IB), ln, q8, vv);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          ww[j] *= v[8 * q8 + j];
          vv[j] *= v[8 * q8 + j];
        }
        row8_put(gen(outb), ln, q8, ww);
        row8_put(gen(outb + OB), ln, q8, vv);
      }
      __syncwarp();
      if (drv.ok) {
        rows_store<T>(gen(outb), static_cast<T*>(q.dv) + o0, ts, row0, Cs, c);
        rows_store<T>(gen(outb + OB), static_cast<T*>(q.dw) + o0, ts, row0, Cs, c);
      }
      __syncwarp();
    }
  }
  cta.finish();
}

// ---------------------------------------------------------------------------
// bwd_grads_kernel: products that contract over the value dimension (K = DV),
// every operand a K-major tile of a [rows][DV] matrix:
//   pass 1: dKs = U dS_C^T, dAs = -P dS_C^T
//   pass 2: dN^qk = dO U^T, dN^qa = -dO P^T, dM^kk = dZ U^T, dM^ka = -dZ P^T (masked)
//   pass 3: dQp = dO S0^T, dKp = dZ S0^T
// ---------------------------------------------------------------------------
template <int DK, int DV, typename T, int NS>
__global__ void __launch_bounds__(256, 1) bwd_grads_kernel(ChunkParams p, BwdBufs q) {
  extern __shared__ __align__(128) uint8_t sm[];
  __shared__ uint64_t bar, bar_cp;
  __shared__ uint32_t tslot;
  const int Cs = p.Cs;
  const SubIdx s = sub_of(p, blockIdx.x, p.nsub, Cs);
  constexpr int NT = 256;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int64_t u = blockIdx.x;
  const uint32_t base = (smem_u32(sm) + 1023u) & ~1023u;  // swizzled tiles start on 1024-byte boundaries
  uint8_t* const sma = sm + (base - smem_u32(sm));
  constexpr uint32_t TB = 128u * 128u * 2u;
  // Every operand is K-major over the DV value columns (rows = tokens or key
  // channels). With DV a multiple of 64 the rows are 128-byte swizzled, so that
  // the row-major staging sweeps store without bank conflicts.
  const auto R0 = kmajor_tile<DV>(base, TB);
  const auto R1 = kmajor_tile<DV>(base + 2 * TB, TB);
  const auto R2 = kmajor_tile<DV>(base + 4 * TB, TB);
  zero_smem(base, 6 * TB);
  if (tid == 0) mbar_init(&bar_cp, 1);
  uint32_t cph = 0;
  TcCta cta;
  cta.init(&tslot, &bar, 512);
  MmaSync drv{&bar, 0u, true};
  const uint32_t lane = tmem_lane_base(warp);
  const int t = tid & 127, wg = tid >> 7;  // TMEM row; warpgroups split the columns
  using RT = std::remove_const_t<decltype(R0)>;
  auto stage_dO = [&](const RT& dst) {  // z * dy (dy alone without z)
    stage_prod<T, false, DV>(dst, p, s, Cs, static_cast<const T*>(p.dy), static_cast<const T*>(p.z), nullptr, 1.f);
  };
  auto stage_U = [&](const RT& dst) {  // w * v
    stage_prod<T, false, DV>(dst, p, s, Cs, static_cast<const T*>(p.v), static_cast<const T*>(p.w), nullptr, 1.f);
  };
  // Rows of a [Cs][N] TMEM result -> dst (fp32, row-major, row stride ld), optional mask.
  float* scratch = reinterpret_cast<float*>(sma + 6 * TB);
  auto drain = [&](uint32_t col, int n, float* dst, int64_t ld, int mask) {
    drain_rows(cta.tmem + lane + 0u, col, n, dst, ld, Cs, scratch, drv.ok, [&](int row, int c, float(&v)[32]) {
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const int sidx = c + j;
        if (mask == 1 && sidx >= row) v[j] = 0.f;  // strictly lower
        if (mask == 2 && sidx > row) v[j] = 0.f;   // lower incl. diagonal
      }
    });
  };
  const uint32_t idK = idesc_bf16(128, DK, 0, 0), idC = idesc_bf16(128, Cs, 0, 0);
  float* g4 = q.g4 + u * 4 * Cs * DK;
  float* dG = q.dG + u * 4 * Cs * Cs;
  const uint32_t mat_dkdv = (uint32_t)DK * DV * 4u, mat_csdv = (uint32_t)Cs * DV * 4u;
  // Each raw fp32 operand is bulk-copied into its tile (raw_issue) while other
  // work runs, and converted once it has landed.
  auto raw_wait = [&] {
    if (!__syncthreads_and(mbar_wait(&bar_cp, cph) ? 1 : 0)) drv.ok = false;
    cph ^= 1u;
  };
  // pass 1: R0 = dS_C, R1 = U, R2 = -P
  fence_async_smem();
  __syncthreads();
  if (tid == 0) mbar_expect_tx(&bar_cp, mat_dkdv + mat_csdv);
  raw_issue(R0, q.dSC + u * DK * DV, DK, DV, &bar_cp);
  raw_issue(R2, q.P + u * Cs * DV, Cs, DV, &bar_cp);
  if (warp < 4) {
    // Everything that reaches the unit's last cumulative log-decay L_{C-1}: the
    // decay of S0 (Gam_C dGam_C, dGam_C = rowsum(dS_C * S0)) plus the suffix
    // factors of K_s and A_s (sum_s K_s dK_s + A_s dA_s, with dK_s = U dS_C^T and
    // dA_s = -P dS_C^T). Since S_C = Diag(Gam_C) S0 + K_s^T U - A_s^T P, the sum
    // is rowsum(dS_C * S_C), with S_C the next unit's start state (or the state
    // after the sequence's last unit). The first four warps take a row at a time,
    // each load reading whole lines, while the other four start staging U.
    const float* d0 = q.dSC + u * DK * DV;
    const float* s0 = s.n + 1 < p.nsub ? q.S_chunks + (u + 1) * DK * DV
                                       : p.S_end + ((int64_t)s.b * p.H + s.h) * DK * DV;
    const int ln = tid & 31;
    constexpr int RB = 8;  // rows per batch of loads
    for (int r0 = warp; r0 < DK; r0 += 4 * RB) {
      float acc[RB];
#pragma unroll
      for (int k = 0; k < RB; ++k) {
        const int row = r0 + 4 * k;
        acc[k] = 0.f;
        if (row < DK && 4 * ln < DV) {
          const float4 a = *reinterpret_cast<const float4*>(d0 + row * DV + 4 * ln);
          const float4 c = *reinterpret_cast<const float4*>(s0 + row * DV + 4 * ln);
          acc[k] = a.x * c.x + a.y * c.y + a.z * c.z + a.w * c.w;
        }
      }
      for (int j = 128; j < DV; j += 128) {  // wider rows than one line per lane
#pragma unroll
        for (int k = 0; k < RB; ++k) {
          const int row = r0 + 4 * k;
          if (row < DK) {
            const float4 a = *reinterpret_cast<const float4*>(d0 + row * DV + j + 4 * ln);
            const float4 c = *reinterpret_cast<const float4*>(s0 + row * DV + j + 4 * ln);
            acc[k] += a.x * c.x + a.y * c.y + a.z * c.z + a.w * c.w;
          }
        }
      }
#pragma unroll
      for (int k = 0; k < RB; ++k) {
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) acc[k] += __shfl_xor_sync(0xffffffffu, acc[k], m);
        const int row = r0 + 4 * k;
        if (ln == 0 && row < DK) q.eC[u * DK + row] = acc[k];
      }
    }
  }
  stage_U(R1);
  raw_wait();
  raw_convert<false>(R0, DK, DV, 1.f);
  raw_convert<false>(R2, Cs, DV, -1.f);
  // TMEM: two pairs of 128-column accumulators, [0, 256) and [256, 512), taken in
  // turn, so that the drain of one pass runs while the tensor core does the next.
  drv.run([&] {
    mma_ops(cta.tmem + 0, kview(R1), kview(R0), DV / 16, idK, NS, false);
    mma_ops(cta.tmem + 128, kview(R2), kview(R0), DV / 16, idK, NS, false);
  });
  // pass 2a: R1 = U, R2 = -P stay; R0 = dO
  stage_dO(R0);
  drv.run_overlap([&] {
                    mma_ops(cta.tmem + 256, kview(R0), kview(R1), DV / 16, idC, NS, false);  // dN^qk
                    mma_ops(cta.tmem + 384, kview(R0), kview(R2), DV / 16, idC, NS, false);  // dN^qa
                  },
                  [&] {
                    drain(0, DK, g4 + 2 * Cs * DK, DK, 0);    // dKs
                    drain(128, DK, g4 + 3 * Cs * DK, DK, 0);  // dAs
                  });
  // pass 2b: R0 = dZ
  if (tid == 0) mbar_expect_tx(&bar_cp, mat_csdv);
  raw_issue(R0, q.dZ + u * Cs * DV, Cs, DV, &bar_cp);
  drain(256, Cs, dG + 2 * Cs * Cs, Cs, 2);
  raw_wait();
  raw_convert<false>(R0, Cs, DV, 1.f);
  drv.run_overlap([&] {
                    mma_ops(cta.tmem + 0, kview(R0), kview(R1), DV / 16, idC, NS, false);    // dM^kk
                    mma_ops(cta.tmem + 128, kview(R0), kview(R2), DV / 16, idC, NS, false);  // dM^ka
                  },
                  [&] { drain(384, Cs, dG + 3 * Cs * Cs, Cs, 2); });
  // pass 3: R0 = dZ stays, R1 = S0, R2 = dO
  if (tid == 0) mbar_expect_tx(&bar_cp, mat_dkdv);
  raw_issue(R1, q.S_chunks + u * DK * DV, DK, DV, &bar_cp);
  stage_dO(R2);
  drain(0, Cs, dG + 0 * Cs * Cs, Cs, 1);
  raw_wait();
  raw_convert<false>(R1, DK, DV, 1.f);
  drv.run_overlap([&] {
                    mma_ops(cta.tmem + 256, kview(R2), kview(R1), DV / 16, idK, NS, false);  // dQp
                    mma_ops(cta.tmem + 384, kview(R0), kview(R1), DV / 16, idK, NS, false);  // dKp
                  },
                  [&] { drain(128, Cs, dG + 1 * Cs * Cs, Cs, 1); });
  drain(256, DK, g4 + 0 * Cs * DK, DK, 0);
  drain(384, DK, g4 + 1 * Cs * DK, DK, 0);
  cta.finish();
}

// ---------------------------------------------------------------------------
// bwd_gram_kernel: the Gram cotangents dG pushed to the Gram factors, per unit
// (sums over the Gram pairs s < t, s <= t for N, channel by channel):
//   dK_left_t  = sum_s (dM^kk_ts k_s + dM^ka_ts a_s) Gam_{t<-s}
//   dQ_left_t  = sum_s (dN^qk_ts k_s + dN^qa_ts a_s) Gam_{t<-s}
//   dK_right_s = sum_t (dM^kk_ts k_t + dN^qk_ts qt_t) Gam_{t<-s}
//   dA_right_s = sum_t (dM^ka_ts k_t + dN^qa_ts qt_t) Gam_{t<-s}
// Pairs across 16-token blocks go level by level as in gram_kernel. With G_b
// the level's tile of dG (row p*2b + X*b + r = (X, t) upper, column
// p*2b + Y*b + r' = (Y, s) lower, zero across pivots):
//   left  phase: D^T = YL^T G_b^T (lane = key channel, column (X, t)), then
//                dX_left_t  += pre16_t F_J(t) D^T[., (X, t)]
//   right phase: D^T = XL^T G_b   (lane = key channel, column (Y, s)), then
//                dY_right_s += suf16_s F_J(s) D^T[., (Y, s)]
// Each phase keeps its levels in TMEM (128 columns each), so every output is
// formed once in the epilogue together with its exact diagonal-block part
// (CUDA cores; the same tree inside the block, down to single tokens) and
// written once.
// ---------------------------------------------------------------------------
// Shared memory of bwd_gram_kernel: the operand and dG tiles, which the
// epilogue reuses for the raw rows of its diagonal blocks (bf16 inputs: k and
// e, or k, g and q, plus log alpha), then the dG diagonal blocks and the tables.
template <int DK>
__host__ __device__ constexpr size_t bwd_gram_front_bytes() {
  constexpr size_t tiles = 2u * 128u * DK * 2u + 2u * 128u * 128u * 2u;
  constexpr size_t rows = 3u * 128u * DK * 2u + 128u * DK * 4u;
  return tiles > rows ? tiles : rows;
}
template <int DK>
__host__ __device__ constexpr size_t bwd_gram_smem_bytes() {
  return 1024u + bwd_gram_front_bytes<DK>() + 8u * SB * SB * 16u + (size_t)kMaxLev * 8u * DK * 4u;
}

template <int DK, typename T, int NS>
__global__ void __launch_bounds__(256, 1) bwd_gram_kernel(ChunkParams p, BwdBufs q) {
  extern __shared__ __align__(128) uint8_t sm[];
  __shared__ uint64_t bar, bar_cp;
  __shared__ uint32_t tslot;
  constexpr int NT = 256;
  const int Cs = p.Cs, nb = Cs / SB, nlev = tree_levels(Cs), lcs = log2_cs(Cs);
  const SubIdx s = sub_of(p, blockIdx.x, p.nsub, Cs);
  const int tid = threadIdx.x, warp = tid >> 5;
  const int64_t u = blockIdx.x;
  const uint32_t base = (smem_u32(sm) + 1023u) & ~1023u;  // swizzled tiles start on 1024-byte boundaries
  uint8_t* const sma = sm + (base - smem_u32(sm));
  constexpr uint32_t OB = 128u * DK * 2u;        // operand tile (128 token rows x dk), one half
  const uint32_t GB = 128u * (uint32_t)Cs * 2u;  // dG tile (128 rows x Cs), one half
  // YL (left phase) or XL (right phase): token rows, read as the MN-major A
  // operand (M = key channel, K = token). With dk a multiple of 64 the rows are
  // 128-byte swizzled, so that the row-major staging sweep stores without bank
  // conflicts; with dk = 32 (rows of 64 bytes) they stay in the no-swizzle layout.
  using OpTile = std::conditional_t<(DK % 64 == 0), SwTile, Tile>;
  OpTile OP;
  if constexpr (DK % 64 == 0) OP = SwTile{base, base + OB, 128u * 128u};
  else OP = Tile{base, base + OB, 128u, DK * 16u};
  const Tile GT{base + 2 * OB, base + 2 * OB + GB, 128u, (uint32_t)Cs * 16u};
  constexpr size_t FB = bwd_gram_front_bytes<DK>();
  float4* dgd = reinterpret_cast<float4*>(sma + FB);  // [nb][16 t][16 s]: mkk, mka, nqk, nqa
  float* ftab = reinterpret_cast<float*>(sma + FB + 8 * SB * SB * 16);  // [kMaxLev][nb][DK]
  constexpr bool kRowsInSmem = sizeof(T) == 2;
  constexpr uint32_t RB = 128u * DK * 2u;  // one bf16 [128][DK] array of raw rows
  const T* rk = reinterpret_cast<const T*>(sma);
  const T* rz1 = reinterpret_cast<const T*>(sma + RB);
  const T* rz2 = reinterpret_cast<const T*>(sma + 2 * RB);
  const float* rla = reinterpret_cast<const float*>(sma + 3 * RB);
  uint32_t cp_phase = 0;
  if (tid == 0) mbar_init(&bar_cp, 1);
  TcCta cta;
  cta.init(&tslot, &bar, tmem_cols_for(128 * nlev));
  MmaSync drv{&bar, 0u, true};
  const float* pre = p.dec + u * 4 * Cs * DK;
  const float* suf = pre + Cs * DK;
  const float* dG = q.dG + u * 4 * Cs * Cs;
  const int64_t gsz = (int64_t)Cs * Cs;
  tree_tables<DK>(pre, ftab, Cs);
#pragma unroll 8
  for (int x = tid; x < nb * SB * SB; x += NT) {  // diagonal blocks of the four cotangents
    const int J = x >> 8, tt = (x >> 4) & 15, ss = x & 15;
    const int64_t o = (int64_t)(SB * J + tt) * Cs + SB * J + ss;
    dgd[x] = make_float4(dG[o], dG[gsz + o], dG[2 * gsz + o], dG[3 * gsz + o]);
  }
  float rv[8];  // r for this thread's 8 channels in stage_level (fixed: 256 pieces per sweep)
  {
    int r_, c8_;
    row_piece<T, DK / 8>(tid, r_, c8_);
    ld8f(p.r + (int64_t)s.h * DK + c8_, rv);
  }
  __syncthreads();

  // G_b, K-major: row (p, X, r) -> t = (2p+1) b + r, column (p', Y, r') -> s = 2p'b + r';
  // dG_{2X+Y}[t][s] when p == p', else 0. Four pieces per thread per batch.
  auto stage_g = [&](int lb) {
    const int b = 1 << lb;
    constexpr int BG = 4;
    for (int x0 = tid; x0 < Cs << (lcs - 3); x0 += BG * NT) {
      Pack8<float> gv[BG];
#pragma unroll
      for (int m = 0; m < BG; ++m) {
        const int x = x0 + m * NT;
        int row, c8;
        piece_of_rt(x, Cs >> 3, row, c8);
        const int pv = row >> (lb + 1), pc = c8 >> (lb + 1);
        if (x < Cs << (lcs - 3) && pv == pc) {
          const int X = (row >> lb) & 1, Y = (c8 >> lb) & 1;
          const int t = (2 * pv + 1) * b + (row & (b - 1)), s0 = 2 * pc * b + (c8 & (b - 1));
          gv[m].ld(dG + (2 * X + Y) * gsz + (int64_t)t * Cs + s0);
        }
      }
#pragma unroll
      for (int m = 0; m < BG; ++m) {
        const int x = x0 + m * NT;
        if (x < Cs << (lcs - 3)) {
          int row, c8;
          piece_of_rt(x, Cs >> 3, row, c8);
          float v[8];
          if ((row >> (lb + 1)) == (c8 >> (lb + 1))) {
            gv[m].get(v);
          } else {
#pragma unroll
            for (int j = 0; j < 8; ++j) v[j] = 0.f;
          }
          put_k(GT, row, c8, v);
        }
      }
    }
  };

  const int i = tid & 127, wg = tid >> 7;  // epilogue: TMEM lane = key channel; warpgroups take alternate blocks
  const int ic = i < DK ? i : DK - 1;
  const int64_t kstride = (int64_t)p.H * DK;
  float* gl = q.gl + u * 4 * Cs * DK;
  for (int side = 0; side < 2 && drv.ok; ++side) {  // 0: left (dK_left, dQ_left), 1: right (dK_right, dA_right)
    const uint32_t id = idesc_bf16(128, Cs, 1, side);
    for (int lev = 0; lev < nlev && drv.ok; ++lev) {
      const int lb = lcs - 1 - lev;
      stage_g(lb);
      stage_level<DK, T>(p, s, pre, suf, ftab + lev * nb * DK, rv, Cs, lb, side == 1, side == 0, OP, OP);
      drv.run([&] {
        if constexpr (DK % 64 == 0)
          mma_ops(cta.tmem + 128 * lev, SwMN{OP}, NoSw{side == 0 ? GT : transposed(GT)}, Cs / 16, id, NS, false);
        else
          mma_tiles(cta.tmem + 128 * lev, transposed(OP), side == 0 ? GT : transposed(GT), Cs / 16, id, NS, false);
      });
    }
    if (!drv.ok) break;
    if constexpr (kRowsInSmem) {
      // raw rows of the unit for the diagonal blocks, one bulk copy per (array, token):
      // left k, e (, -), log alpha; right k, g, q, log alpha
      const int na = side == 0 ? 2 : 3;
      fence_async_smem();
      __syncthreads();
      const bool no_g = side == 1 && !p.g;  // static-only readout: g = 1 is not copied
      if (tid == 0) mbar_expect_tx(&bar_cp, (uint32_t)Cs * DK * (2u * (na - (no_g ? 1 : 0)) + 4u));
      for (int x = tid; x < Cs * 4; x += NT) {
        const int a = x / Cs, tok = x % Cs;
        const int64_t o = toff(p, s.b, s.tok0 + tok, s.h, DK);
        if (a < na && !(no_g && a == 1)) {
          const void* src = a == 0 ? p.k : (side == 0 ? p.e : (a == 1 ? p.g : p.q));
          bulk_g2s(base + a * RB + tok * DK * 2, static_cast<const T*>(src) + o, DK * 2, &bar_cp);
        } else if (a == 3) {
          bulk_g2s(base + 3 * RB + tok * DK * 4, p.la + o, DK * 4, &bar_cp);
        }
      }
      if (no_g) {  // the g rows are ones
        const uint4 one = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
        for (uint32_t o = tid * 16u; o < (uint32_t)Cs * DK * 2u; o += NT * 16u) sts128(base + RB + o, one);
      }
      const bool ok = mbar_wait(&bar_cp, cp_phase);
      cp_phase ^= 1u;
      if (!__syncthreads_and(ok ? 1 : 0)) drv.ok = false;
      if (!drv.ok) break;
    }
    for (int J = wg; J < nb; J += 2) {
      float acc[2][SB];
#pragma unroll
      for (int c = 0; c < 2; ++c)
#pragma unroll
        for (int tt = 0; tt < SB; ++tt) acc[c][tt] = 0.f;
      for (int lev = 0; lev < nlev; ++lev) {
        const int lb = lcs - 1 - lev, b = 1 << lb;
        const bool upper = ((SB * J) >> lb) & 1;
        if (upper != (side == 0)) continue;  // warp-uniform
        const int pv = (SB * J) >> (lb + 1);
        const int r0 = SB * J - (upper ? (2 * pv + 1) * b : 2 * pv * b);
        const float f = ftab[(lev * nb + J) * DK + ic];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          float v[16];
          tmem_ld16(cta.tmem + tmem_lane_base(warp) + 128 * lev + pv * 2 * b + c * b + r0, v);
#pragma unroll
          for (int tt = 0; tt < SB; ++tt) acc[c][tt] += f * v[tt];
        }
      }
      if (i >= DK) continue;
      float K[SB], Z[SB], al[SB];  // Z = a (left) or qt (right)
      const float rr = p.r[(int64_t)s.h * DK + i];
      if constexpr (kRowsInSmem) {
#pragma unroll
        for (int tt = 0; tt < SB; ++tt) {
          const int ro = (SB * J + tt) * DK + i;
          const float kk = __bfloat162float(rk[ro]);
          K[tt] = kk;
          Z[tt] = side == 0 ? __bfloat162float(rz1[ro]) * kk : rr * __bfloat162float(rz1[ro]) * __bfloat162float(rz2[ro]);
          al[tt] = expf(rla[ro]);
        }
      } else {
        const int64_t o0 = toff(p, s.b, s.tok0 + SB * J, s.h, DK) + i;
#pragma unroll
        for (int tt = 0; tt < SB; ++tt) {
          const int64_t o = o0 + tt * kstride;
          const float kk = Elt<T>::ld(static_cast<const T*>(p.k) + o);
          K[tt] = kk;
          Z[tt] = side == 0 ? Elt<T>::ld(static_cast<const T*>(p.e) + o) * kk
                            : rr * Elt<T>::ld_or_one(p.g ? static_cast<const T*>(p.g) + o : nullptr) *
                                  Elt<T>::ld(static_cast<const T*>(p.q) + o);
          al[tt] = expf(__ldg(p.la + o));
        }
      }
      // the block-relative decay products of these 16 tokens, formed from their
      // alphas in the decay kernel's order (so equal to its pre and suf tables):
      // pre_t from the block start through t (left phase), suf_s over the tokens
      // after s to the block end (right phase)
      if (side == 0) {
        float run = 1.f;
#pragma unroll
        for (int tt = 0; tt < SB; ++tt) {
          run *= al[tt];
          acc[0][tt] *= run;
          acc[1][tt] *= run;
        }
      } else {
        float run = 1.f;
#pragma unroll
        for (int tt = SB - 1; tt >= 0; --tt) {
          acc[0][tt] *= run;
          acc[1][tt] *= run;
          run *= al[tt];
        }
      }
      // Diagonal block, exact: pairs ss < tt inside the block go by sub-pivots
      // (halves of 8, 4, 2, 1 tokens), where Gam_{tt<-ss} = fac_tt * fac_ss with
      // fac the running product from the sub-pivot forward (upper tt) or backward
      // (lower ss); the pairs tt == ss have Gam = 1.
      const float4* dg = dgd + J * SB * SB;
#pragma unroll
      for (int tt = 0; tt < SB; ++tt) {  // tt == ss
        const float4 g = dg[tt * SB + tt];
        if (side == 0) {
          acc[0][tt] += g.x * K[tt] + g.y * Z[tt];
          acc[1][tt] += g.z * K[tt] + g.w * Z[tt];
        } else {
          acc[0][tt] += g.x * K[tt] + g.z * Z[tt];
          acc[1][tt] += g.y * K[tt] + g.w * Z[tt];
        }
      }
#pragma unroll
      for (int sl = 0; sl < 4; ++sl) {
        const int hb = 8 >> sl;  // half-length of this sub-level
        float fac[SB], sk[SB], sz[SB];
#pragma unroll
        for (int b0 = 0; b0 < SB; b0 += 2 * hb) {
          float run = 1.f;
#pragma unroll
          for (int uu = b0 + hb; uu < b0 + 2 * hb; ++uu) {  // upper: from the sub-pivot forward
            run *= al[uu];
            fac[uu] = run;
          }
          run = 1.f;
#pragma unroll
          for (int uu = b0 + hb - 1; uu >= b0; --uu) {  // lower: from the sub-pivot backward
            fac[uu] = run;
            run *= al[uu];
          }
        }
#pragma unroll
        for (int uu = 0; uu < SB; ++uu) {
          sk[uu] = K[uu] * fac[uu];
          sz[uu] = Z[uu] * fac[uu];
        }
#pragma unroll
        for (int b0 = 0; b0 < SB; b0 += 2 * hb) {
          if (side == 0) {
#pragma unroll
            for (int tt = b0 + hb; tt < b0 + 2 * hb; ++tt) {
              float a0 = 0.f, a1 = 0.f;
#pragma unroll
              for (int ss = b0; ss < b0 + hb; ++ss) {
                const float4 g = dg[tt * SB + ss];
                a0 += g.x * sk[ss] + g.y * sz[ss];  // dK_left
                a1 += g.z * sk[ss] + g.w * sz[ss];  // dQ_left
              }
              acc[0][tt] += fac[tt] * a0;
              acc[1][tt] += fac[tt] * a1;
            }
          } else {
#pragma unroll
            for (int ss = b0; ss < b0 + hb; ++ss) {
              float a0 = 0.f, a1 = 0.f;
#pragma unroll
              for (int tt = b0 + hb; tt < b0 + 2 * hb; ++tt) {
                const float4 g = dg[tt * SB + ss];
                a0 += g.x * sk[tt] + g.z * sz[tt];  // dK_right
                a1 += g.y * sk[tt] + g.w * sz[tt];  // dA_right
              }
              acc[0][ss] += fac[ss] * a0;
              acc[1][ss] += fac[ss] * a1;
            }
          }
        }
      }
#pragma unroll
      for (int tt = 0; tt < SB; ++tt) {
        const int64_t o = (int64_t)(SB * J + tt) * DK + i;
        gl[(2 * side + 0) * Cs * DK + o] = acc[0][tt];
        gl[(2 * side + 1) * Cs * DK + o] = acc[1][tt];
      }
    }
    __syncthreads();  // the raw rows are read; the next phase restages over them
  }
  cta.finish();
}

// ---------------------------------------------------------------------------
// bwd_final_kernel: per unit, thread = key channel i:
//   dL_t = k dKl + qt dQl - k dKr - a dAr + Kp dKp + Qp dQp - Ks dKs - As dAs
//   dL_{C-1} += sum_s (Ks dKs + As dAs) + Gam_C dGam_C = rowsum(dS_C * S_C)
//   dlog_alpha_t = sum_{u >= t} dL_u
//   dqt = dQl + Gam dQp, da = dAr + Gsuf dAs, dk = dKl + dKr + Gam dKp + Gsuf dKs + e da
//   dq = r g dqt, dg = r q dqt, dr += g q dqt, de = k da  (dv, dw come from bwd_dz)
// ---------------------------------------------------------------------------
template <int DK, int DV, typename T>
__global__ void __launch_bounds__(128) bwd_final_kernel(ChunkParams p, BwdBufs q) {
  const int Cs = p.Cs;
  const int64_t u = blockIdx.x;
  const SubIdx s = sub_of(p, (int)u, p.nsub, Cs);
  const int i = threadIdx.x;
  const int64_t stride_k = (int64_t)p.H * DK;
  if (i < DK) {
    const float* gam = p.dec + (u * 4 + 2) * Cs * DK;
    const float* gsuf = p.dec + (u * 4 + 3) * Cs * DK;
    const float* g4 = q.g4 + u * 4 * Cs * DK;
    const float* gl = q.gl + u * 4 * Cs * DK;
    const float rr = p.r[(int64_t)s.h * DK + i];
    const int64_t o0 = toff(p, s.b, s.tok0, s.h, DK) + i;
    // what lands on the last token's cumulative log-decay enters every dlog_alpha
    // of the unit (gathered by bwd_grads)
    const float E = __ldg(q.eC + u * DK + i);
    float run = E, dr_acc = 0.f;
#pragma unroll 8
    for (int tt = Cs - 1; tt >= 0; --tt) {
      const int64_t o = o0 + tt * stride_k;
      const float kk = Elt<T>::ld(static_cast<const T*>(p.k) + o);
      const float ee = Elt<T>::ld(static_cast<const T*>(p.e) + o);
      const float gg = Elt<T>::ld_or_one(p.g ? static_cast<const T*>(p.g) + o : nullptr);
      const float qq = Elt<T>::ld(static_cast<const T*>(p.q) + o);
      const float a = ee * kk, qt = rr * gg * qq;
      const int ti = tt * DK + i;
      const float G = __ldg(gam + ti), Gs = __ldg(gsuf + ti);
      const float dQp = __ldg(g4 + 0 * Cs * DK + ti), dKp = __ldg(g4 + 1 * Cs * DK + ti);
      const float dKs = __ldg(g4 + 2 * Cs * DK + ti), dAs = __ldg(g4 + 3 * Cs * DK + ti);
      const float dKl = __ldg(gl + 0 * Cs * DK + ti), dQl = __ldg(gl + 1 * Cs * DK + ti);
      const float dKr = __ldg(gl + 2 * Cs * DK + ti), dAr = __ldg(gl + 3 * Cs * DK + ti);
      run += kk * dKl + qt * dQl - kk * dKr - a * dAr + kk * G * dKp + qt * G * dQp - kk * Gs * dKs - a * Gs * dAs;
      q.dla[o] = run;
      const float dqt = dQl + G * dQp;
      const float da = dAr + Gs * dAs;
      const float dkt = dKl + dKr + G * dKp + Gs * dKs + ee * da;
      Elt<T>::st(static_cast<T*>(q.dq) + o, rr * gg * dqt);
      if (q.dg) Elt<T>::st(static_cast<T*>(q.dg) + o, rr * qq * dqt);
      Elt<T>::st(static_cast<T*>(q.dk) + o, dkt);
      Elt<T>::st(static_cast<T*>(q.de) + o, kk * da);
      dr_acc += gg * qq * dqt;
    }
    if (q.dr) atomicAdd(q.dr + (int64_t)s.h * DK + i, dr_acc);
  }
}

}  // namespace muir
