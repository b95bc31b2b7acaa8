// Single-token recurrent step (streaming decode) and state initialisation.
//
// One CTA owns one (row n, head h, 32-column slab of the state). The slab's
// dk x 32 fp32 tile is read once into registers as float4s, decayed, reduced
// column-wise (prediction p_j and readout partial sums) with warp shuffles plus
// a small shared-memory exchange, updated and written back once. Every value
// column j of the update depends only on column j of S, so slabs are
// independent and the state is touched exactly twice (one read, one write).
//
//   p_j   = sum_i alpha_i S_ij k_i
//   sig_j = sum_i alpha_i S_ij qt_i
//   S'_ij = alpha_i S_ij - a_i p_j + k_i u_j            (a = e*k, u = w*v)
//   o_j   = sum_i S'_ij qt_i = sig_j - p_j (a.qt) + u_j (k.qt)
//   y_j   = z_j o_j
#pragma once

#include "common.cuh"

namespace muir {

struct DecodeParams {
  int64_t n_seq;
  int H, dk, dv;
  float* S;
  const void *q, *k, *v, *e, *w, *g, *z;
  const float* la;
  const float* r;
  int64_t r_stride;
  void* y;
};

template <int DK, typename T>
__global__ void __launch_bounds__(128) decode_step_kernel(DecodeParams p) {
  constexpr int RM = DK / 16;  // rows per thread
  const int tid = threadIdx.x;
  const int cg = tid & 7;      // column group: 4 columns
  const int rg = tid >> 3;     // row group: rows rg, rg+16, ...
  const int slabs = p.dv >> 5;
  const int64_t blk = blockIdx.x;
  const int slab = (int)(blk % slabs);
  const int64_t nh = blk / slabs;
  const int h = (int)(nh % p.H);
  const int64_t n = nh / p.H;

  __shared__ float s_k[DK], s_a[DK], s_q[DK], s_al[DK];
  __shared__ float s_u[32], s_z[32];
  __shared__ float s_red[2][4][32];
  __shared__ float s_dot[2][4];

  // Issue the state loads first: they are the only large transfer.
  float* Sb = p.S + (nh * DK) * (int64_t)p.dv + slab * 32 + cg * 4;
  float4 x[RM];
#pragma unroll
  for (int m = 0; m < RM; ++m)
    x[m] = *reinterpret_cast<const float4*>(Sb + (int64_t)(rg + 16 * m) * p.dv);

  // Per-row vectors of this (n, h).
  const int64_t vo = nh * DK;
  float kq = 0.f, aq = 0.f;
  for (int i = tid; i < DK; i += 128) {
    const float kk = Elt<T>::ld(static_cast<const T*>(p.k) + vo + i);
    const float ee = Elt<T>::ld(static_cast<const T*>(p.e) + vo + i);
    const float gg = Elt<T>::ld_or_one(p.g ? static_cast<const T*>(p.g) + vo + i : nullptr);
    const float qq = Elt<T>::ld(static_cast<const T*>(p.q) + vo + i);
    const float rr = __ldg(p.r + n * p.r_stride + (int64_t)h * DK + i);
    const float al = expf(__ldg(p.la + vo + i));
    const float qt = rr * gg * qq;
    const float a = ee * kk;
    s_k[i] = kk; s_a[i] = a; s_q[i] = qt; s_al[i] = al;
    kq += kk * qt;
    aq += a * qt;
  }
  kq = warp_sum(kq);
  aq = warp_sum(aq);
  if ((tid & 31) == 0) { s_dot[0][tid >> 5] = kq; s_dot[1][tid >> 5] = aq; }
  if (tid < 32) {
    const int64_t co = nh * (int64_t)p.dv + slab * 32 + tid;
    s_u[tid] = Elt<T>::ld(static_cast<const T*>(p.w) + co) * Elt<T>::ld(static_cast<const T*>(p.v) + co);
    s_z[tid] = p.z ? Elt<T>::ld(static_cast<const T*>(p.z) + co) : 1.f;
  }
  __syncthreads();

  float p1[4] = {0.f, 0.f, 0.f, 0.f}, p2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int m = 0; m < RM; ++m) {
    const int i = rg + 16 * m;
    const float al = s_al[i], kk = s_k[i], qt = s_q[i];
    x[m].x *= al; x[m].y *= al; x[m].z *= al; x[m].w *= al;
    p1[0] += x[m].x * kk; p1[1] += x[m].y * kk; p1[2] += x[m].z * kk; p1[3] += x[m].w * kk;
    p2[0] += x[m].x * qt; p2[1] += x[m].y * qt; p2[2] += x[m].z * qt; p2[3] += x[m].w * qt;
  }
  // Reduce over the 16 row groups: 4 inside the warp (lanes differing in bits 3,4), 4 warps via smem.
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    p1[c] += __shfl_xor_sync(0xffffffffu, p1[c], 8);
    p1[c] += __shfl_xor_sync(0xffffffffu, p1[c], 16);
    p2[c] += __shfl_xor_sync(0xffffffffu, p2[c], 8);
    p2[c] += __shfl_xor_sync(0xffffffffu, p2[c], 16);
  }
  const int warp = tid >> 5, lane = tid & 31;
  if (lane < 8) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      s_red[0][warp][lane * 4 + c] = p1[c];
      s_red[1][warp][lane * 4 + c] = p2[c];
    }
  }
  __syncthreads();
  float pj[4], sj[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const int j = cg * 4 + c;
    pj[c] = s_red[0][0][j] + s_red[0][1][j] + s_red[0][2][j] + s_red[0][3][j];
    sj[c] = s_red[1][0][j] + s_red[1][1][j] + s_red[1][2][j] + s_red[1][3][j];
  }
  float uj[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) uj[c] = s_u[cg * 4 + c];
#pragma unroll
  for (int m = 0; m < RM; ++m) {
    const int i = rg + 16 * m;
    const float a = s_a[i], kk = s_k[i];
    float4 o;
    o.x = x[m].x - a * pj[0] + kk * uj[0];
    o.y = x[m].y - a * pj[1] + kk * uj[1];
    o.z = x[m].z - a * pj[2] + kk * uj[2];
    o.w = x[m].w - a * pj[3] + kk * uj[3];
    *reinterpret_cast<float4*>(Sb + (int64_t)i * p.dv) = o;
  }
  if (tid < 8) {
    const float KQ = s_dot[0][0] + s_dot[0][1] + s_dot[0][2] + s_dot[0][3];
    const float AQ = s_dot[1][0] + s_dot[1][1] + s_dot[1][2] + s_dot[1][3];
    float yo[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) yo[c] = s_z[cg * 4 + c] * (sj[c] - pj[c] * AQ + uj[c] * KQ);
    Elt<T>::st4(static_cast<T*>(p.y) + nh * (int64_t)p.dv + slab * 32 + cg * 4, yo);
  }
}

// Row energies of states S [n,H,dk,dv] -> r[h,i] = (mean_{n,j} S[n,h,i,j]^2 + eps)^(-exponent).
// One CTA per (h, i); the sum of squares is accumulated in fp64.
__global__ void row_scale_kernel(const float* __restrict__ S, int64_t n, int H, int dk, int dv, float exponent,
                                 float eps, float* __restrict__ r) {
  const int h = blockIdx.x / dk, i = blockIdx.x % dk;
  double acc = 0.0;
  const int64_t per = n * dv;
  for (int64_t x = threadIdx.x; x < per; x += blockDim.x) {
    const int64_t m = x / dv, j = x % dv;
    const float v = __ldg(S + (((m * H + h) * dk + i) * dv + j));
    acc += (double)v * v;
  }
  __shared__ double part[32];
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double tot = 0.0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) tot += part[w];
    const double e = tot / (double)per + (double)eps;
    r[(int64_t)h * dk + i] = (float)pow(e, -(double)exponent);
  }
}

__global__ void state_init_kernel(float4* __restrict__ S, const float4* __restrict__ src, int64_t n4) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n4; i += (int64_t)gridDim.x * blockDim.x)
    S[i] = src ? src[i] : make_float4(0.f, 0.f, 0.f, 0.f);
}

}  // namespace muir
