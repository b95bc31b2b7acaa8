// Chunkwise-parallel forward pass of the Muir gated delta rule.
//
// Notation for one chunk of C tokens (local index t = 0..C-1) with start state
// S0, per (batch, head):
//   Gam_{t<-s} = prod_{u=s+1..t} alpha_u (per key channel), Gam_t = prod_{u<=t},
//   Gsuf_t = prod_{u>t} (to the chunk end), Gam_C = prod over the chunk.
//   K, A = e*k, Qt = r*g*q (key rows), U = w*v (value columns).
//   M^kk_ts = k_t.Gam_{t<-s}.k_s, M^ka_ts = k_t.Gam_{t<-s}.a_s          (s < t)
//   N^qk_ts = qt_t.Gam_{t<-s}.k_s, N^qa_ts = qt_t.Gam_{t<-s}.a_s        (s <= t)
//   T = (I + M^ka)^-1,  W = T (K*Gam),  Ut = T M^kk U
//   Phi  = Diag(Gam_C) - (A*Gsuf)^T W            (dk x dk)
//   Psi  = (K*Gsuf)^T U - (A*Gsuf)^T Ut          (dk x dv)
//   Q'   = Qt*Gam - N^qa W                        (C x dk)
//   Oloc = N^qk U - N^qa Ut                       (C x dv)
// and the chunk acts on the state as an affine map:
//   S_C = Phi S0 + Psi,   O = Q' S0 + Oloc,   y = z * O.
// (Derivation: unroll the recurrence inside the chunk; the prediction vector P
// of all tokens solves (I + M^ka) P = (K*Gam) S0 + M^kk U.)
//
// Decay products are boundary-pivoted (openai-hub article, section on the TPU
// chunkwise algorithm; liuch.name post, third bullet): the chunk is cut into
// blocks of SB = 16 tokens. For s in block I and t in a later block J,
//   Gam_{t<-s} = suf_s * mid(I,J) * pre_t
// with suf_s = prod_{u=s+1..end(I)}, pre_t = prod_{u=start(J)..t} and mid the
// product of whole blocks in between: every factor is a product of alphas, so
// it lies in [0, 1] and nothing is divided. Off-diagonal Gram blocks then are
// tensor-core GEMMs of pivot-scaled operands; the diagonal blocks (8x8 in the
// forward Grams, 16x16 in their backward) are computed exactly on the CUDA
// cores with running products.
//
// Kernels (one CTA per (batch, head, unit of Cs = min(chunk, 128) tokens) unless noted):
//   decay_kernel      pre, suf, Gam_t, Gsuf_t            -> workspace
//                     (a thread per 16-token block and key channel)
//   gram_kernel       the 4 Grams (gram.cuh): blocks across the binary tree of
//                     8-token blocks on tcgen05 (one product per level), the
//                     exact 8x8 diagonal blocks on the CUDA cores meanwhile
//   solve_kernel      T: exact 16x16 leaves, then recursive 2x2 block merges
//                     T21 = -T22 M21 T11 on tcgen05 (block-Neumann recursion)
//   maps_kernel       W, Ut, Phi, Psi, Q', Oloc (tcgen05)  -> workspace
//   compose_kernel    (chunk 256) composes two 128-token half-chunk maps
//   scan_kernel       sequential over chunks per (batch, head, kSlab-column slab):
//                     S_C = Phi S0 + Psi (tcgen05), states -> workspace
//   out_kernel        chunk-parallel y = z * (Q' S0 + Oloc) (tcgen05)
#pragma once

#include "tc.cuh"

namespace muir {

constexpr int SB = 16;  // pivot block length (tokens)

// Column slab width of the sequential scans: Psi (and the backward's E) are
// stored per unit as [dv / kSlab][dk][kSlab], and every scan CTA carries one
// kSlab-column slab of the state, so that B * H * dv / kSlab CTAs run the scan.
constexpr int kSlab = 16;
__host__ __device__ inline int64_t slab_off(int c, int row, int dk) {
  return ((int64_t)(c / kSlab) * dk + row) * kSlab + (c % kSlab);
}

struct ChunkParams {
  int B;
  int64_t T;
  int H, dk, dv;
  int Cs;    // tokens per local unit (min(chunk, 128))
  int nsub;  // T / Cs
  int C;     // chunk length of the state scan (Cs or 2*Cs)
  const void *q, *k, *v, *e, *w, *g, *z;
  const float* la;
  const float* r;
  const float* S0;
  // workspace
  float* dec;  // [nsubtot][4][Cs][dk]: pre, suf, Gam, Gsuf
  uint8_t* gr; // [nsubtot][4] images of M^kk, M^ka, N^qk, N^qa (see sq_put)
  uint8_t* tt; // [nsubtot] image of T
  uint8_t* ma;  // [nunits] images of Phi and Q' (see MapGeom)
  float* psi;   // [nunits][dv/kSlab][dk][kSlab]: Psi in column slabs (slab_off)
  float* ol;    // [nunits][Cs][dv]: Oloc
  uint8_t* ma2; // the same three for chunk-256 maps composed from two 128-token units
  float* psi2;
  float* ol2;   // [nunits/2][256][dv]
  // outputs
  void* y;
  float* S_T;
  float* S_chunks;  // optional [units][dk][dv]: state at the start of every unit
  float* S_end;     // optional [B*H][dk][dv]: state after the last unit (kept for the backward)
  // backward
  float* wsave;     // optional [nsubtot][Cs][dk]: W
  float* usave;     // optional [nsubtot][Cs][dv]: Ut
  const void* dy;   // [B,T,H,dv]
  void* dz;         // [B,T,H,dv] or null
};

struct SubIdx {
  int b, h, n;
  int64_t tok0;
};

__device__ __forceinline__ SubIdx sub_of(const ChunkParams& p, int sid, int units_per_seq, int unit_len) {
  SubIdx s;
  s.n = sid % units_per_seq;
  const int bh = sid / units_per_seq;
  s.h = bh % p.H;
  s.b = bh / p.H;
  s.tok0 = (int64_t)s.n * unit_len;
  return s;
}

// Offset of element 0 of token `tok` of (b, h) in a [B,T,H,d] tensor.
__device__ __forceinline__ int64_t toff(const ChunkParams& p, int b, int64_t tok, int h, int d) {
#ifdef MUIR_CHECK
  if (!check_bounds(b >= 0 && b < p.B && tok >= 0 && tok < p.T && h >= 0 && h < p.H, kStatusBoundsToken)) return 0;
#endif
  return (((int64_t)b * p.T + tok) * p.H + h) * d;
}

__device__ __forceinline__ void ld8f(const float* p, float (&o)[8]) { Elt<float>::ld8(p, o); }

// N consecutive floats from shared memory (p aligned to 4 * min(N, 4) bytes), vectorised.
template <int N>
__device__ __forceinline__ void lds_vec(const float* p, float (&o)[N]) {
  if constexpr (N % 4 == 0) {
#pragma unroll
    for (int i = 0; i < N / 4; ++i) {
      const float4 a = reinterpret_cast<const float4*>(p)[i];
      o[4 * i] = a.x; o[4 * i + 1] = a.y; o[4 * i + 2] = a.z; o[4 * i + 3] = a.w;
    }
  } else if constexpr (N == 1) {
    o[0] = *p;
  } else {
    static_assert(N % 2 == 0, "even length");
#pragma unroll
    for (int i = 0; i < N / 2; ++i) {
      const float2 a = reinterpret_cast<const float2*>(p)[i];
      o[2 * i] = a.x; o[2 * i + 1] = a.y;
    }
  }
}

__device__ __forceinline__ Tile sub_tile(const Tile& t, int k0, int mn0) {
  const uint32_t off = (uint32_t)(k0 >> 3) * t.lbo + (uint32_t)(mn0 >> 3) * t.sbo;
  return Tile{t.hi + off, t.lo + off, t.lbo, t.sbo};
}

__device__ __forceinline__ void zero_smem(uint32_t base, uint32_t bytes) {
  const uint4 z = make_uint4(0, 0, 0, 0);
  for (uint32_t o = threadIdx.x * 16u; o < bytes; o += blockDim.x * 16u) sts128(base + o, z);
}

__device__ __forceinline__ uint32_t tmem_cols_for(int n) {
  return n <= 32 ? 32u : n <= 64 ? 64u : n <= 128 ? 128u : n <= 256 ? 256u : 512u;
}

// Workspace image of a chunk map with L tokens: tile 0 holds Phi (dk x dk),
// tiles 1.. hold Q' (128 token rows each). Every tile is a bf16 hi block then a
// lo block of 128 rows x dk in the K-major canonical layout (sbo = dk*16),
// exactly as the MMA reads it, so consumers fetch tiles with bulk copies.
struct MapGeom {
  int ntile;      // 1 + ceil(L / 128)
  uint32_t half;  // bytes of one hi (or lo) block
  uint32_t tile;  // hi + lo
  uint32_t unit;  // all tiles of one map
};
__host__ __device__ inline MapGeom map_geom(int dk, int L) {
  MapGeom g;
  g.ntile = 1 + (L + 127) / 128;
  g.half = 128u * (uint32_t)dk * 2u;
  g.tile = 2u * g.half;
  g.unit = (uint32_t)g.ntile * g.tile;
  return g;
}

// Row i of Phi, 8 consecutive columns c8.., as bf16 hi/lo.
__device__ __forceinline__ void map_put_phi(uint8_t* img, const MapGeom& g, int dk, int i, int c8, const float (&x)[8]) {
  gput_k(img, g.half, (uint32_t)dk * 16u, i, c8, x);
}
// Row t (token) of Q'.
__device__ __forceinline__ void map_put_q(uint8_t* img, const MapGeom& g, int dk, int t, int c8, const float (&x)[8]) {
  gput_k(img + (uint32_t)(1 + (t >> 7)) * g.tile, g.half, (uint32_t)dk * 16u, t & 127, c8, x);
}

// Workspace image of a Cs x Cs matrix (a Gram or T): bf16 hi block then lo
// block of 128 rows x Cs columns in the K-major canonical layout (sbo = Cs*16),
// row = first index. Consumers bulk-copy it; a K-major read contracts over the
// columns, the transposed view (lbo = Cs*16, sbo = 128) over the rows.
__host__ __device__ inline uint32_t sq_half(int Cs) { return 128u * (uint32_t)Cs * 2u; }
__host__ __device__ inline uint32_t sq_bytes(int Cs) { return 2u * sq_half(Cs); }
__device__ __forceinline__ void sq_put(uint8_t* img, int Cs, int r, int c8, const float (&x)[8]) {
#ifdef MUIR_CHECK
  if (!check_bounds(r >= 0 && r < Cs && c8 >= 0 && c8 + 8 <= Cs, kStatusBoundsImage)) return;
#endif
  gput_k(img, sq_half(Cs), (uint32_t)Cs * 16u, r, c8, x);
}
// An image is lower block-triangular: in row group rg (rows 8 rg .. + 7) only
// the columns up to the end of the diagonal 16-block, 16 (rg / 2 + 1), can be
// nonzero, and they are the first sq_prefix(rg) bytes of the group's Cs * 16.
__host__ __device__ inline uint32_t sq_prefix(int rg) { return (uint32_t)(2 * (rg >> 1) + 2) * 128u; }
// zeroed shared-memory source of the bulk stores that clear the rest (>= Cs * 16 - 256)
constexpr uint32_t kZeroBuf = 2048u;
__device__ __forceinline__ float sq_get(const uint8_t* img, int Cs, int r, int c) {
  const uint32_t off = (uint32_t)(r >> 3) * (uint32_t)Cs * 16u + (uint32_t)(c >> 3) * 128u + (uint32_t)(r & 7) * 16u +
                       (uint32_t)(c & 7) * 2u;
  const __nv_bfloat16 h = *reinterpret_cast<const __nv_bfloat16*>(img + off);
  const __nv_bfloat16 l = *reinterpret_cast<const __nv_bfloat16*>(img + sq_half(Cs) + off);
  return __bfloat162float(h) + __bfloat162float(l);
}

// Bulk copy of `bytes` (multiple of 16) in pieces of at most 32 KB.
__device__ __forceinline__ void bulk_g2s_big(uint32_t dst, const uint8_t* src, uint32_t bytes, uint64_t* bar) {
  for (uint32_t o = 0; o < bytes; o += 32768u) {
    const uint32_t n = bytes - o < 32768u ? bytes - o : 32768u;
    bulk_g2s(dst + o, src + o, n, bar);
  }
}

// Stage a contiguous fp32 matrix src[rows][cols] (rows a multiple of 8, cols / 8
// a power of two, rows * cols <= 128 * 128) times `sign` as a bf16 hi/lo operand
// tile: K-major over cols (put_k, row = MN index) or, with MN, MN-major over rows
// (put_mn, row = K index). The raw matrix arrives by bulk copy into the tile's
// own shared memory (hi and lo halves contiguous, at least 4 bytes per element),
// every thread takes its pieces into registers, and after a barrier writes them
// back converted. In two steps: raw_issue (thread 0 starts the copy on `bar`,
// whose transaction count the caller has set) and, once the copy has landed,
// raw_convert (every thread; ends without a barrier). stage_raw does both.
template <typename OpTile>
__device__ __forceinline__ void raw_issue(const OpTile& t, const float* src, int rows, int cols, uint64_t* bar) {
  if (threadIdx.x == 0)
    bulk_g2s_big(t.hi, reinterpret_cast<const uint8_t*>(src), (uint32_t)rows * (uint32_t)cols * 4u, bar);
}
template <bool MN, typename OpTile>
__device__ __forceinline__ void raw_convert(const OpTile& t, int rows, int cols, float sign) {
  constexpr int NT = 256, MAXP = 128 * 128 / 8 / NT;
  const float4* raw = reinterpret_cast<const float4*>(__cvta_shared_to_generic(t.hi));
  const int np = rows * cols / 8;
  const int g = cols / 8;
  float v[MAXP][8];
#pragma unroll
  for (int k = 0; k < MAXP; ++k) {
    const int x = threadIdx.x + k * NT;
    if (x < np) {
      int r, c8;
      if constexpr (std::is_same_v<OpTile, SwTile>) piece_of_swz(x, g, r, c8);
      else piece_of_rot(x, g, r, c8);
      const int e = r * g + (c8 >> 3);
      const float4 a = raw[2 * e], b = raw[2 * e + 1];
      v[k][0] = sign * a.x; v[k][1] = sign * a.y; v[k][2] = sign * a.z; v[k][3] = sign * a.w;
      v[k][4] = sign * b.x; v[k][5] = sign * b.y; v[k][6] = sign * b.z; v[k][7] = sign * b.w;
    }
  }
  __syncthreads();
#pragma unroll
  for (int k = 0; k < MAXP; ++k) {
    const int x = threadIdx.x + k * NT;
    if (x < np) {
      int r, c8;
      if constexpr (std::is_same_v<OpTile, SwTile>) piece_of_swz(x, g, r, c8);
      else piece_of_rot(x, g, r, c8);
      if constexpr (MN) put_mn(t, r, c8, v[k]);
      else put_op(t, r, c8, v[k]);
    }
  }
}
// 256 threads, all of which call it; no MMA may be reading the tile. Returns
// false if the copy's bounded wait ran out.
template <bool MN>
__device__ __forceinline__ bool stage_raw(const Tile& t, const float* src, int rows, int cols, float sign,
                                          uint64_t* bar, uint32_t& phase) {
  fence_async_smem();
  __syncthreads();
  if (threadIdx.x == 0) mbar_expect_tx(bar, (uint32_t)rows * (uint32_t)cols * 4u);
  raw_issue(t, src, rows, cols, bar);
  const bool ok = __syncthreads_and(mbar_wait(bar, phase) ? 1 : 0) != 0;
  phase ^= 1u;
  raw_convert<MN>(t, rows, cols, sign);
  return ok;
}

// Stage the elementwise product a * b * f * sign over the unit's `rows` tokens as
// a bf16 hi/lo operand tile (rows = tokens): K-major over the COLS channels
// (put_k) or, with MN, MN-major with K = token (put_mn). a, b are [B,T,H,COLS]
// inputs (b may be null), f a contiguous fp32 [rows][COLS] matrix (may be
// null). 256 threads; BT tokens per thread per batch with every load of a batch
// issued before any is used.
template <typename T, bool MN, int COLS, typename OpTile>
__device__ __forceinline__ void stage_prod(const OpTile& t, const ChunkParams& p, const SubIdx& s, int rows,
                                           const T* a, const T* b, const float* f, float sign) {
  constexpr int NT = 256, BT = sizeof(T) == 2 ? 4 : 2, G = COLS / 8;
  for (int x0 = threadIdx.x; x0 < rows * G; x0 += BT * NT) {
    Pack8<T> pa[BT], pb[BT];
    Pack8<float> pf[BT];
#pragma unroll
    for (int u = 0; u < BT; ++u) {
      const int x = x0 + u * NT;
      if (x < rows * G) {
        int r, c8;
        row_piece<T, G>(x, r, c8);
        const int64_t o = toff(p, s.b, s.tok0 + r, s.h, COLS) + c8;
        pa[u].ld(a + o);
        if (b) pb[u].ld(b + o);
        if (f) pf[u].ld(f + r * COLS + c8);
      }
    }
#pragma unroll
    for (int u = 0; u < BT; ++u) {
      const int x = x0 + u * NT;
      if (x < rows * G) {
        int r, c8;
        row_piece<T, G>(x, r, c8);
        float va[8], vb[8];
        pa[u].get(va);
        if (b) {
          pb[u].get(vb);
#pragma unroll
          for (int j = 0; j < 8; ++j) va[j] *= vb[j];
        }
        if (f) {
          pf[u].get(vb);
#pragma unroll
          for (int j = 0; j < 8; ++j) va[j] *= vb[j];
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) va[j] *= sign;
        if constexpr (MN) put_mn(t, r, c8, va);
        else put_op(t, r, c8, va);
      }
    }
  }
}

// Bytes of shared scratch drain_rows needs: 32 x 32 floats for each of 8 warps.
constexpr uint32_t kDrainScratch = 8u * 32u * 32u * 4u;

// Drain TMEM columns [col, col + n) (n a multiple of 32) of this warp's 32 rows
// (TMEM lanes 32 (w % 4) ..; the two warpgroups take alternate 32-column chunks)
// to the row-major fp32 matrix dst (row stride ld floats, rows 16-byte aligned).
// A row-per-lane store would touch 32 lines per instruction; instead each chunk
// goes through this warp's 4 KB of `scratch` (16-byte piece j of row r at piece
// j ^ (r & 7), conflict-free both ways) and out as 4 rows x 128 bytes per
// store. mask(row, c, v) may edit the 32 values first. Rows >= nrows, and all
// rows when !on, are not stored. Every thread calls it.
template <typename F>
__device__ __forceinline__ void drain_rows(uint32_t tmem_lane_addr, uint32_t col, int n, float* dst, int64_t ld,
                                           int nrows, float* scratch, bool on, F mask) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, wg = w >> 2;
  const int row0 = (w & 3) * 32;
  float* sc = scratch + w * 32 * 32;
  for (int c = wg * 32; c < n; c += 64) {
    float v[32];
    tmem_ld32(tmem_lane_addr + col + c, v);
    mask(row0 + lane, c, v);
#pragma unroll
    for (int j = 0; j < 8; ++j)
      *reinterpret_cast<float4*>(sc + lane * 32 + ((j ^ (lane & 7)) << 2)) =
          make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
    __syncwarp();
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int r = (lane >> 3) + 4 * i, j = lane & 7;
      const float4 a = *reinterpret_cast<const float4*>(sc + r * 32 + ((j ^ (r & 7)) << 2));
      if (on && row0 + r < nrows) *reinterpret_cast<float4*>(dst + (int64_t)(row0 + r) * ld + c + 4 * j) = a;
    }
    __syncwarp();
  }
}

// ---- 32 x 32 row blocks through a per-warp scratch ---------------------------
// An epilogue thread owns one row (its TMEM lane), so a thread-per-row load or
// store of a row-major matrix touches 32 lines per instruction. These helpers
// move the 32 rows [row0, row0 + 32) x columns [c, c + 32) that a warp owns in
// whole lines instead: 16-byte asynchronous copies (cp.async) into a scratch
// block, and stores of 4 rows x 128 bytes (fp32) or 8 rows x 64 bytes (bf16)
// per instruction out of it. In an fp32 block (4 KB) the 16-byte piece j of row
// r sits at piece j ^ (r & 7); in a bf16 block (2 KB) piece q of row r at
// q ^ (r & 3): conflict-free for the row-wise and the line-wise accesses alike.
// Rows >= nrows are neither loaded nor stored.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

template <typename T>
constexpr uint32_t row_block_bytes() { return sizeof(T) == 4 ? 4096u : 2048u; }

template <typename T>
__device__ __forceinline__ void rows_fill(uint32_t blk, const T* src, int64_t ld, int row0, int nrows, int c) {
  const int lane = threadIdx.x & 31;
  if constexpr (sizeof(T) == 4) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int r = (lane >> 3) + 4 * i, j = lane & 7;
      if (row0 + r < nrows)
        cp_async16(blk + (uint32_t)(r * 128 + ((j ^ (r & 7)) << 4)), src + (int64_t)(row0 + r) * ld + c + 4 * j);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = (lane >> 2) + 8 * i, q = lane & 3;
      if (row0 + r < nrows)
        cp_async16(blk + (uint32_t)(r * 64 + ((q ^ (r & 3)) << 4)), src + (int64_t)(row0 + r) * ld + c + 8 * q);
    }
  }
}

// Columns 8q .. 8q+7 of row r of a block, as floats.
template <typename T>
__device__ __forceinline__ void row8_get(const uint8_t* blk, int r, int q, float (&o)[8]) {
  if constexpr (sizeof(T) == 4) {
    const float4 a = *reinterpret_cast<const float4*>(blk + r * 128 + (((2 * q) ^ (r & 7)) << 4));
    const float4 b = *reinterpret_cast<const float4*>(blk + r * 128 + (((2 * q + 1) ^ (r & 7)) << 4));
    o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w; o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
  } else {
    Pack8<__nv_bfloat16> pk;
    pk.u = *reinterpret_cast<const uint4*>(blk + r * 64 + ((q ^ (r & 3)) << 4));
    pk.get(o);
  }
}
__device__ __forceinline__ void row8_put(uint8_t* blk, int r, int q, const float (&v)[8]) {
  *reinterpret_cast<float4*>(blk + r * 128 + (((2 * q) ^ (r & 7)) << 4)) = make_float4(v[0], v[1], v[2], v[3]);
  *reinterpret_cast<float4*>(blk + r * 128 + (((2 * q + 1) ^ (r & 7)) << 4)) = make_float4(v[4], v[5], v[6], v[7]);
}

// An fp32 block out to the row-major matrix dst (element type T) in whole lines.
template <typename T>
__device__ __forceinline__ void rows_store(const uint8_t* blk, T* dst, int64_t ld, int row0, int nrows, int c) {
  const int lane = threadIdx.x & 31;
  if constexpr (sizeof(T) == 4) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int r = (lane >> 3) + 4 * i, j = lane & 7;
      const float4 a = *reinterpret_cast<const float4*>(blk + r * 128 + ((j ^ (r & 7)) << 4));
      if (row0 + r < nrows) *reinterpret_cast<float4*>(dst + (int64_t)(row0 + r) * ld + c + 4 * j) = a;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = (lane >> 2) + 8 * i, q = lane & 3;
      float v[8];
      row8_get<float>(blk, r, q, v);
      if (row0 + r < nrows) Elt<T>::st8(dst + (int64_t)(row0 + r) * ld + c + 8 * q, v);
    }
  }
}

// CTA prologue shared by the tensor-core kernels: TMEM allocation + mbarrier.
struct TcCta {
  uint32_t tmem;
  uint32_t ncols;
  __device__ __forceinline__ void init(uint32_t* slot, uint64_t* bar, uint32_t cols) {
    ncols = cols;
    if ((threadIdx.x >> 5) == 0) tmem_alloc(slot, cols);
    if (threadIdx.x == 0) mbar_init(bar, 1);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    tmem = *slot;
  }
  __device__ __forceinline__ void finish() {
    tc_fence_before();
    __syncthreads();
    if ((threadIdx.x >> 5) == 0) tmem_dealloc(tmem, ncols);
  }
};

// Input row helpers: 8 consecutive channels of token `tok`.
template <typename T>
struct Rows {
  const ChunkParams& p;
  int b, h;
  __device__ __forceinline__ void k(int64_t tok, int c8, float (&o)[8]) const {
    Elt<T>::ld8(static_cast<const T*>(p.k) + toff(p, b, tok, h, p.dk) + c8, o);
  }
  __device__ __forceinline__ void a(int64_t tok, int c8, float (&o)[8]) const {
    float kk[8], ee[8];
    Elt<T>::ld8(static_cast<const T*>(p.k) + toff(p, b, tok, h, p.dk) + c8, kk);
    Elt<T>::ld8(static_cast<const T*>(p.e) + toff(p, b, tok, h, p.dk) + c8, ee);
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] = ee[i] * kk[i];
  }
  __device__ __forceinline__ void qt(int64_t tok, int c8, float (&o)[8]) const {
    float qq[8], gg[8], rr[8];
    Elt<T>::ld8(static_cast<const T*>(p.q) + toff(p, b, tok, h, p.dk) + c8, qq);
    if (p.g) {
      Elt<T>::ld8(static_cast<const T*>(p.g) + toff(p, b, tok, h, p.dk) + c8, gg);
    } else {  // static-only readout: g = 1
#pragma unroll
      for (int i = 0; i < 8; ++i) gg[i] = 1.f;
    }
    ld8f(p.r + (int64_t)h * p.dk + c8, rr);
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] = rr[i] * gg[i] * qq[i];
  }
  __device__ __forceinline__ void u(int64_t tok, int c8, float (&o)[8]) const {
    float vv[8], ww[8];
    Elt<T>::ld8(static_cast<const T*>(p.v) + toff(p, b, tok, h, p.dv) + c8, vv);
    Elt<T>::ld8(static_cast<const T*>(p.w) + toff(p, b, tok, h, p.dv) + c8, ww);
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] = ww[i] * vv[i];
  }
};

// ---------------------------------------------------------------------------
// decay_kernel: one CTA per unit, thread = (16-token block, key channel).
//   pre[t]  = prod_{u=start(block)..t} alpha_u     suf[t]  = prod_{u=t+1..end(block)} alpha_u
//   gam[t]  = prod_{u=0..t} alpha_u               gsuf[t] = prod_{u=t+1..Cs-1} alpha_u
// built as running products of alphas inside blocks and products of whole-block
// totals across blocks (no division, every factor in [0, 1]). Each thread walks
// its block's 16 tokens; the block totals meet in shared memory, and the
// products across blocks are taken in token order (before a block) and in
// reverse token order (after it).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) decay_kernel(ChunkParams p) {
  __shared__ float tot[8][128];  // block totals: Cs / 16 <= 8 blocks, dk <= 128 channels
  const int dk = p.dk, Cs = p.Cs, nb = Cs / SB;
  const SubIdx s = sub_of(p, blockIdx.x, p.nsub, Cs);
  const int i = threadIdx.x % dk, jb = threadIdx.x / dk;
  const bool on = jb < nb;
  float* pre = p.dec + (int64_t)blockIdx.x * 4 * Cs * dk;
  float* suf = pre + Cs * dk;
  float* gam = suf + Cs * dk;
  float* gsuf = gam + Cs * dk;
  const int64_t stride = (int64_t)p.H * dk;
  const float* la = p.la + toff(p, s.b, s.tok0 + (on ? jb * SB : 0), s.h, dk) + i;
  float a[SB], pr[SB];
  float run = 1.f;
  if (on) {
#pragma unroll
    for (int u = 0; u < SB; ++u) a[u] = expf(__ldg(la + u * stride));
#pragma unroll
    for (int u = 0; u < SB; ++u) {
      run *= a[u];
      pr[u] = run;
      pre[(jb * SB + u) * dk + i] = run;
    }
    tot[jb][i] = run;
  }
  __syncthreads();
  if (!on) return;
  float before = 1.f, after = 1.f;
  for (int J = 0; J < jb; ++J) before *= tot[J][i];
  for (int J = nb - 1; J > jb; --J) after *= tot[J][i];
  float srun = 1.f;
#pragma unroll
  for (int u = SB - 1; u >= 0; --u) {
    const int o = (jb * SB + u) * dk + i;
    gam[o] = before * pr[u];
    suf[o] = srun;
    gsuf[o] = srun * after;
    srun *= a[u];
  }
}

// ---------------------------------------------------------------------------
// Levels of the binary tree over a unit's 16-token blocks (shared by the Gram
// kernel and its backward). Level lev has half-length b = Cs >> (lev + 1)
// (64, 32, 16 for Cs = 128) and pivots P = (2p+1) b; tokens t with (t / b) odd
// are "upper" (t >= P), the others "lower" (t < P).
// ---------------------------------------------------------------------------
constexpr int kMaxLev = 3;
__device__ __forceinline__ int tree_levels(int Cs) { return Cs == 128 ? 3 : 2; }
__device__ __forceinline__ int log2_cs(int Cs) { return Cs == 128 ? 7 : 6; }

// ftab[lev][J][i] = F^b_J: product of the block totals between block J and its
// pivot (upper blocks: pivot block .. J-1; lower blocks: J+1 .. pivot block - 1).
// pre is the unit's in-block prefix product (pre[16 J + 15] = total of block J).
template <int DK>
__device__ __forceinline__ void tree_tables(const float* pre, float* ftab, int Cs) {
  const int nb = Cs / SB, nlev = tree_levels(Cs), i = threadIdx.x;
  if (i < DK) {
    float tot[8];
#pragma unroll
    for (int J = 0; J < 8; ++J) tot[J] = J < nb ? pre[(SB * J + SB - 1) * DK + i] : 1.f;
    for (int lev = 0; lev < nlev; ++lev) {
      const int hb = (Cs >> (lev + 1)) / SB;  // blocks per half
      for (int J0 = 0; J0 < nb; J0 += 2 * hb) {
        float run = 1.f;
        for (int J = J0 + hb; J < J0 + 2 * hb; ++J) {  // upper half: from the pivot forward
          ftab[(lev * nb + J) * DK + i] = run;
          run *= tot[J];
        }
        run = 1.f;
        for (int J = J0 + hb - 1; J >= J0; --J) {  // lower half: from the pivot backward
          ftab[(lev * nb + J) * DK + i] = run;
          run *= tot[J];
        }
      }
    }
  }
}

// Operands of level lev (b = 2^lb):
//   XL row p*2b + X*b + r = [k; r g q]_t * pre_t * F_J(t)   upper t = (2p+1)b + r
//   YL row p*2b + Y*b + r = [k; e k]_s  * suf_s * F_J(s)    lower s = 2pb + r
// Staged for the halves asked for; 256 threads, BT tokens per thread per batch
// with all loads of a batch issued before any is used. Pieces go by row_piece,
// which keeps a thread on the same 8 channels throughout: rv holds r there.
// The operand tiles are no-swizzle Tiles (put_k) or SwTiles (put_sw).

template <int DK, typename T, typename OpTile>
__device__ __forceinline__ void stage_level(const ChunkParams& p, const SubIdx& s, const float* pre,
                                            const float* suf, const float* ft, const float (&rv)[8], int Cs,
                                            int lb, bool want_upper, bool want_lower, const OpTile& XL,
                                            const OpTile& YL) {
  constexpr int NT = 256;
  constexpr int BT = sizeof(T) == 2 ? 4 : 2;
  const int b = 1 << lb;
  for (int x0 = threadIdx.x; x0 < Cs * (DK / 8); x0 += BT * NT) {
    Pack8<T> pk[BT], p1[BT], p2[BT];
    Pack8<float> ps[BT];
#pragma unroll
    for (int u = 0; u < BT; ++u) {
      const int x = x0 + u * NT;
      int t, c8;
      row_piece<T, DK / 8>(x, t, c8);
      const bool upper = (t >> lb) & 1;
      if (x < Cs * (DK / 8) && (upper ? want_upper : want_lower)) {
        const int64_t o = toff(p, s.b, s.tok0 + t, s.h, DK) + c8;
        pk[u].ld(static_cast<const T*>(p.k) + o);
        p1[u].ld(static_cast<const T*>(upper ? p.q : p.e) + o);
        p2[u].ld(static_cast<const T*>(upper && p.g ? p.g : p.k) + o);
        ps[u].ld((upper ? pre : suf) + t * DK + c8);
      }
    }
#pragma unroll
    for (int u = 0; u < BT; ++u) {
      const int x = x0 + u * NT;
      int t, c8;
      row_piece<T, DK / 8>(x, t, c8);
      const bool upper = (t >> lb) & 1;
      if (x < Cs * (DK / 8) && (upper ? want_upper : want_lower)) {
        const int pv = t >> (lb + 1), r = t & (b - 1);
        float kk[8], s1[8], s2[8], sc[8], fj[8];
        pk[u].get(kk);
        p1[u].get(s1);
        p2[u].get(s2);
        ps[u].get(sc);
        if (upper && !p.g) {  // static-only readout: g = 1 (p2 held k as a stand-in)
#pragma unroll
          for (int j = 0; j < 8; ++j) s2[j] = 1.f;
        }
        Elt<float>::ld8g(ft + (t >> 4) * DK + c8, fj);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float f = sc[j] * fj[j];
          s1[j] *= s2[j] * (upper ? rv[j] : 1.f) * f;  // r g q or e k
          kk[j] *= f;
        }
        const OpTile& dst = upper ? XL : YL;
        put_op(dst, (pv << (lb + 1)) + r, c8, kk);
        put_op(dst, (pv << (lb + 1)) + b + r, c8, s1);
      }
    }
  }
}

// ---------------------------------------------------------------------------
// solve_kernel: T = (I + M^ka)^-1 (unit lower triangular) by the recursive
// block method: exact 16x16 leaves by forward substitution, then for block size
// h = 16, 32, 64 every pair [[A,0],[B,D]] of adjacent h-blocks gets the lower
// left block -D^-1 B A^-1 = -T_D (M_B T_A): two batches of tcgen05 MMAs per
// level (X = M_B T_A, then Y = T_D X).
// ---------------------------------------------------------------------------
template <int NS>
__global__ void __launch_bounds__(256, 1) solve_kernel(ChunkParams p) {
  extern __shared__ __align__(128) uint8_t sm[];
  __shared__ uint64_t bar, bar_cp;
  __shared__ uint32_t tslot;
  const int Cs = p.Cs, nb = Cs / SB;
  constexpr int NT = 256;
  const int tid = threadIdx.x, warp = tid >> 5;
  const uint32_t H = sq_half(Cs);
  const uint32_t base = smem_u32(sm);
  const Tile TM{base, base + H, 128u, (uint32_t)Cs * 16u};                 // M^ka image, K-major
  const Tile TA{base + 2 * H, base + 3 * H, 128u, (uint32_t)Cs * 16u};     // T so far, K-major
  const Tile TBt{base + 4 * H, base + 5 * H, 128u, (uint32_t)Cs * 16u};    // T so far / X, MN-major
  float* leaf = reinterpret_cast<float*>(sm + 6 * H);                      // [nb][16][16]
  const uint8_t* smc = sm;
  if (tid == 0) mbar_init(&bar_cp, 1);
  zero_smem(base + 2 * H, 4 * H);
  TcCta cta;
  cta.init(&tslot, &bar, 256);
  if (tid == 0) {
    mbar_expect_tx(&bar_cp, 2 * H);
    bulk_g2s_big(base, p.gr + ((int64_t)blockIdx.x * 4 + 1) * sq_bytes(Cs), 2 * H, &bar_cp);
  }
  MmaSync drv{&bar, 0u, true};
  drv.ok = __syncthreads_and(mbar_wait(&bar_cp, 0) ? 1 : 0) != 0;
  // exact 16x16 leaves: column j of (I + M_JJ)^-1 by forward substitution
  {
    const int J = tid >> 4, j = tid & 15;
    if (J < nb) {
      float x[SB];
#pragma unroll
      for (int i = 0; i < SB; ++i) x[i] = (i == j) ? 1.f : 0.f;
#pragma unroll
      for (int i = 1; i < SB; ++i) {
        float acc = 0.f;
#pragma unroll
        for (int kk = 0; kk < i; ++kk) acc += sq_get(smc, Cs, SB * J + i, SB * J + kk) * x[kk];
        if (i > j) x[i] = -acc;
      }
#pragma unroll
      for (int i = 0; i < SB; ++i) leaf[(J * SB + i) * SB + j] = x[i];
    }
  }
  __syncthreads();
  for (int x = tid; x < nb * SB * 2; x += NT) {  // leaves -> both tiles
    const int J = x / (SB * 2), i = (x / 2) % SB, c8 = (x & 1) * 8;
    float v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = leaf[(J * SB + i) * SB + c8 + e];
    put_k(TA, SB * J + i, SB * J + c8, v);
    put_mn(TBt, SB * J + i, SB * J + c8, v);
  }
  const int t = tid & 127, wg = tid >> 7;
  for (int h = SB; h < Cs && drv.ok; h *= 2) {
    // X = M (K-range = the even block) * T_even: only rows of the odd block are used
    const int nm = Cs / (2 * h);
    const uint32_t idh = idesc_bf16(128, h, 0, 1);
    drv.run([&] {
      for (int m = 0; m < nm; ++m)
        mma_tiles(cta.tmem + 2 * m * h, sub_tile(TM, 2 * m * h, 0), sub_tile(TBt, 2 * m * h, 2 * m * h), h / 16, idh,
                  NS, false);
    });
    if (!drv.ok) break;
    const int m = t / (2 * h);
    const bool odd = t < Cs && ((t / h) & 1);
    for (int c = wg * 16; c < h; c += 32) {  // X (odd rows, even-block columns) -> B tile
      float v[16];
      tmem_ld16(cta.tmem + tmem_lane_base(warp) + 2 * m * h + c, v);
      if (odd) {
        float a[8], b8[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) { a[j] = v[j]; b8[j] = v[8 + j]; }
        put_mn(TBt, t, 2 * m * h + c, a);
        put_mn(TBt, t, 2 * m * h + c + 8, b8);
      }
    }
    drv.run([&] {
      for (int mm = 0; mm < nm; ++mm)
        mma_tiles(cta.tmem + 128 + 2 * mm * h, sub_tile(TA, (2 * mm + 1) * h, 0),
                  sub_tile(TBt, (2 * mm + 1) * h, 2 * mm * h), h / 16, idh, NS, false);
    });
    if (!drv.ok) break;
    for (int c = wg * 16; c < h; c += 32) {  // new lower-left block -T_odd X into both tiles
      float v[16];
      tmem_ld16(cta.tmem + tmem_lane_base(warp) + 128 + 2 * m * h + c, v);
      if (odd) {
        float a[8], b8[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) { a[j] = -v[j]; b8[j] = -v[8 + j]; }
        put_k(TA, t, 2 * m * h + c, a);
        put_k(TA, t, 2 * m * h + c + 8, b8);
        put_mn(TBt, t, 2 * m * h + c, a);
        put_mn(TBt, t, 2 * m * h + c + 8, b8);
      }
    }
  }
  fence_async_smem();
  __syncthreads();
  // the K-major tile of T is exactly its workspace image: one bulk store
  if (drv.ok && tid == 0) {
    uint8_t* out = p.tt + (int64_t)blockIdx.x * sq_bytes(Cs);
    for (uint32_t o = 0; o < 2 * H; o += 32768u) bulk_s2g(out + o, base + 2 * H + o, 2 * H - o < 32768u ? 2 * H - o : 32768u);
    bulk_commit();
    bulk_wait_all();
  }
  cta.finish();
}

// ---------------------------------------------------------------------------
// maps_kernel: the chunk's affine map. TMEM column bases (fp32, 128 lanes):
//   phase 1: W -> 0, Z = M^kk U -> 128, Ut = T Z -> 256
//   phase 2: Phi -> 384, Psi -> 128 (Z consumed)
//   phase 3: Oloc -> 256 (Ut consumed), Q' -> 0 (W consumed)
// Shared memory: one A tile and two MN-major B tiles (128 x 128 bf16 hi+lo
// each). Negated operands are staged negated. The MN-major tiles the threads
// stage (B1, B2, and A when it holds (X*Gsuf)^T) leave 16 bytes between the
// 8-column blocks (SBO = Cs*16 + 16): the staging sweep reads token rows whole,
// and the 8 threads of a shared-memory phase, which store 8 consecutive column
// blocks of one row, then land in 8 distinct bank groups.
// ---------------------------------------------------------------------------
constexpr uint32_t kMapsPlane = 128u * 128u * 2u + 16u * 16u;  // one padded bf16 plane, at most 16 column blocks
constexpr size_t maps_smem_bytes() { return 6u * kMapsPlane; }

template <int DK, int DV, typename T, int NS>
__global__ void __launch_bounds__(256, 1) maps_kernel(ChunkParams p) {
  extern __shared__ __align__(128) uint8_t sm[];
  __shared__ uint64_t bar, bar_cp;
  __shared__ uint32_t tslot;
  const int Cs = p.Cs;
  const SubIdx s = sub_of(p, blockIdx.x, p.nsub, Cs);
  constexpr int NT = 256;
  const int tid = threadIdx.x, warp = tid >> 5;
  constexpr uint32_t TBP = kMapsPlane;
  static_assert(DK <= 128 && DV <= 128, "maps tiles hold at most 16 column blocks");
  const uint32_t base = smem_u32(sm);
  const uint32_t kstride = (uint32_t)Cs * 16u;  // every tile here contracts over the Cs tokens
  const uint32_t kpad = kstride + 16u;          // column-block stride of the thread-staged tiles
  const uint32_t H = sq_half(Cs);
  const Tile A{base, base + H, 128u, kstride};  // bulk-copied Gram / T image
  const Tile As{base, base + TBP, 128u, kpad};  // the same memory holding a staged (X*Gsuf)^T
  const Tile B1{base + 2 * TBP, base + 3 * TBP, 128u, kpad};
  const Tile B2{base + 4 * TBP, base + 5 * TBP, 128u, kpad};
  if (tid == 0) mbar_init(&bar_cp, 1);
  zero_smem(base + 2 * TBP, 4 * TBP);
  TcCta cta;
  cta.init(&tslot, &bar, 512);
  const float* dec = p.dec + (int64_t)blockIdx.x * 4 * Cs * DK;
  const float* gam = dec + 2 * Cs * DK;
  const float* gsuf = dec + 3 * Cs * DK;
  const uint8_t* G = p.gr + (int64_t)blockIdx.x * 4 * sq_bytes(Cs);
  const uint8_t* Tm = p.tt + (int64_t)blockIdx.x * sq_bytes(Cs);
  MmaSync drv{&bar, 0u, true};
  const uint32_t lane = tmem_lane_base(warp);
  const int t = tid & 127, wg = tid >> 7;  // TMEM row; warpgroups take alternate 16-column chunks
  // W stays in TMEM until its second use; Z's and Ut's columns are reused once they are consumed
  constexpr uint32_t cW = 0, cZ = 128, cUt = 256, cPhi = 384, cPsi = 128, cOl = 256, cQ = 0;
  uint32_t cp_phase = 0;
  // A <- a Gram or T image (one bulk copy); the MMA that last read A has completed.
  // issue_img starts the copy, wait_img waits for it: work that does not touch A
  // can run in between.
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
  // TMEM columns [col, col+n) of this thread's row (times sign) -> MN-major B tile row t.
  auto tmem_to_b = [&](const Tile& dst, uint32_t col, int n, float sign) {
    for (int c = wg * 16; c < n; c += 32) {
      float v[16];
      tmem_ld16(cta.tmem + lane + col + c, v);
      if (t < Cs) {
        float a[8], b8[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) { a[j] = sign * v[j]; b8[j] = sign * v[8 + j]; }
        put_mn(dst, t, c, a);
        put_mn(dst, t, c + 8, b8);
      }
    }
  };
  // (X * Gsuf)^T as an MN-major A operand (M = channel, K = token), X = k or e k, scaled by sign.
  auto stage_suffixed = [&](bool erase, float sign) {
    stage_prod<T, true, DK>(As, p, s, Cs, static_cast<const T*>(p.k), erase ? static_cast<const T*>(p.e) : nullptr,
                            gsuf, sign);
  };
  const uint32_t idK = idesc_bf16(128, DK, 0, 1), idV = idesc_bf16(128, DV, 0, 1);
  const uint32_t idKt = idesc_bf16(128, DK, 1, 1), idVt = idesc_bf16(128, DV, 1, 1);
  // ---- phase 1: W = T (K*Gam), Z = M^kk U, Ut = T Z
  issue_img(Tm);
  stage_prod<T, true, DK>(B1, p, s, Cs, static_cast<const T*>(p.k), nullptr, gam, 1.f);  // K*Gam (K = token)
  stage_prod<T, true, DV>(B2, p, s, Cs, static_cast<const T*>(p.v), static_cast<const T*>(p.w), nullptr, 1.f);  // U
  wait_img();
  drv.run([&] { mma_tiles(cta.tmem + cW, A, B1, Cs / 16, idK, NS, false); });
  load_img(G + 0 * sq_bytes(Cs));  // M^kk
  drv.run([&] { mma_tiles(cta.tmem + cZ, A, B2, Cs / 16, idV, NS, false); });
  issue_img(Tm);
  tmem_to_b(B1, cZ, DV, 1.f);
  wait_img();
  drv.run([&] { mma_tiles(cta.tmem + cUt, A, B1, Cs / 16, idV, NS, false); });
  auto no_mask = [](int, int, float(&)[32]) {};
  if (p.wsave) {  // the backward pass reuses W and Ut: out in whole lines through
                  // the A tile's memory (its last product has completed)
    float* wo = p.wsave + (int64_t)blockIdx.x * Cs * DK;
    float* uo = p.usave + (int64_t)blockIdx.x * Cs * DV;
    float* scr = reinterpret_cast<float*>(sm);
    drain_rows(cta.tmem + lane, cW, DK, wo, DK, Cs, scr, drv.ok, no_mask);
    drain_rows(cta.tmem + lane, cUt, DV, uo, DV, Cs, scr, drv.ok, no_mask);
    __syncthreads();  // the scratch is read before (X*Gsuf)^T is staged over it
  }
  // ---- phase 2, A = (A*Gsuf)^T staged once for both of its products:
  //   D_Phi = (A*Gsuf)^T W (Phi = Diag(Gam_C) - D_Phi in the epilogue), Psi = (A*Gsuf)^T (-Ut) + (K*Gsuf)^T U
  tmem_to_b(B1, cW, DK, 1.f);
  stage_suffixed(true, 1.f);
  drv.run([&] { mma_tiles(cta.tmem + cPhi, As, B1, Cs / 16, idKt, NS, false); });
  tmem_to_b(B1, cUt, DV, -1.f);
  drv.run([&] { mma_tiles(cta.tmem + cPsi, As, B1, Cs / 16, idVt, NS, false); });
  stage_suffixed(false, 1.f);
  drv.run([&] { mma_tiles(cta.tmem + cPsi, As, B2, Cs / 16, idVt, NS, true); });
  // ---- phase 3: Oloc = N^qa (-Ut) + N^qk U, and N^qa W (Q' = Qt*Gam - N^qa W in the epilogue)
  load_img(G + 3 * sq_bytes(Cs));  // N^qa
  drv.run([&] { mma_tiles(cta.tmem + cOl, A, B1, Cs / 16, idV, NS, false); });  // B1 holds -Ut
  tmem_to_b(B1, cW, DK, 1.f);
  drv.run([&] { mma_tiles(cta.tmem + cQ, A, B1, Cs / 16, idK, NS, false); });
  issue_img(G + 2 * sq_bytes(Cs));  // N^qk (A is free: the Q product has completed)
  // Qt * Gam (Qt = r g q) as fp32 rows in B1's shared memory (B1 is free), read
  // back by the epilogue's TMEM rows. The 16-byte chunk j of row t is stored at
  // chunk j ^ (t & 7), so that 8 consecutive rows reading the same chunk hit 8
  // distinct bank groups.
  float* qgam = reinterpret_cast<float*>(sm + 2 * TBP);
  {
    constexpr int BT = 4;
    const T* gp = static_cast<const T*>(p.g);
    for (int x0 = tid; x0 < Cs * (DK / 8); x0 += BT * NT) {
      Pack8<T> pq[BT], pg[BT];
      Pack8<float> pm[BT];
#pragma unroll
      for (int u = 0; u < BT; ++u) {
        const int x = x0 + u * NT;
        if (x < Cs * (DK / 8)) {
          const int r = x / (DK / 8), c8 = (x % (DK / 8)) * 8;
          const int64_t o = toff(p, s.b, s.tok0 + r, s.h, DK) + c8;
          pq[u].ld(static_cast<const T*>(p.q) + o);
          pg[u].ld_or_one(gp ? gp + o : nullptr);  // static-only readout: g = 1
          pm[u].ld(gam + r * DK + c8);
        }
      }
#pragma unroll
      for (int u = 0; u < BT; ++u) {
        const int x = x0 + u * NT;
        if (x < Cs * (DK / 8)) {
          const int r = x / (DK / 8), c8 = (x % (DK / 8)) * 8;
          float qq[8], gg[8], gm[8], rr[8];
          pq[u].get(qq);
          pg[u].get(gg);
          pm[u].get(gm);
          ld8f(p.r + (int64_t)s.h * DK + c8, rr);
#pragma unroll
          for (int j = 0; j < 8; ++j) qq[j] = (rr[j] * gg[j] * qq[j]) * gm[j];
          const int j0 = c8 >> 2;
          *reinterpret_cast<float4*>(qgam + r * DK + ((j0 ^ (r & 7)) << 2)) = make_float4(qq[0], qq[1], qq[2], qq[3]);
          *reinterpret_cast<float4*>(qgam + r * DK + (((j0 + 1) ^ (r & 7)) << 2)) =
              make_float4(qq[4], qq[5], qq[6], qq[7]);
        }
      }
    }
  }
  wait_img();
  drv.run([&] { mma_tiles(cta.tmem + cOl, A, B2, Cs / 16, idV, NS, true); });
  // ---- epilogue: Phi, Q' -> map image (bf16 hi/lo tiles); Psi -> 32-column slabs; Oloc -> row-major
  const MapGeom mg = map_geom(DK, Cs);
  uint8_t* ma = p.ma + (int64_t)blockIdx.x * mg.unit;
  float* psi = p.psi + (int64_t)blockIdx.x * DK * DV;
  float* ol = p.ol + (int64_t)blockIdx.x * Cs * DV;
  const float* gC = gam + (Cs - 1) * DK;
  for (int c = wg * 16; c < DK; c += 32) {
    float v[16];
    tmem_ld16(cta.tmem + lane + cPhi + c, v);
    if (t < DK && drv.ok) {
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        v[j] = -v[j];
        if (c + j == t) v[j] += gC[t];
      }
      float a8[8], b8[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) { a8[j] = v[j]; b8[j] = v[8 + j]; }
      map_put_phi(ma, mg, DK, t, c, a8);
      map_put_phi(ma, mg, DK, t, c + 8, b8);
    }
  }
  for (int c = wg * 16; c < DV; c += 32) {
    float v[16];
    tmem_ld16(cta.tmem + lane + cPsi + c, v);
    if (t < DK && drv.ok) {
      float* o = psi + slab_off(c, t, DK);
      stg_row16(o, v);
    }
  }
  // Q' = Qt * Gam - N^qa W, Qt * Gam from shared memory (staged above)
  for (int c = wg * 16; c < DK; c += 32) {
    float v[16];
    tmem_ld16(cta.tmem + lane + cQ + c, v);
    if (t < Cs && drv.ok) {
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const float4 a = *reinterpret_cast<const float4*>(qgam + t * DK + ((((c >> 2) + jj) ^ (t & 7)) << 2));
        v[4 * jj] = a.x - v[4 * jj];
        v[4 * jj + 1] = a.y - v[4 * jj + 1];
        v[4 * jj + 2] = a.z - v[4 * jj + 2];
        v[4 * jj + 3] = a.w - v[4 * jj + 3];
      }
      float a8[8], b8[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) { a8[j] = v[j]; b8[j] = v[8 + j]; }
      map_put_q(ma, mg, DK, t, c, a8);
      map_put_q(ma, mg, DK, t, c + 8, b8);
    }
  }
  // Oloc out in whole lines through B2's memory (its last product has completed)
  drain_rows(cta.tmem + lane, cOl, DV, ol, DV, Cs, reinterpret_cast<float*>(sm + 4 * TBP), drv.ok, no_mask);
  cta.finish();
}

// ---------------------------------------------------------------------------
// compose_kernel (chunk = 256): the map of a 256-token chunk from the maps of
// its two 128-token halves (h0 then h1), which is the top-level merge of the
// recursive block solve applied to the chunk map:
//   Phi = Phi1 Phi0,  Psi = Phi1 Psi0 + Psi1
//   first-half outputs: Q'0, Oloc0 (unchanged)
//   second-half outputs: Q'1 Phi0, Q'1 Psi0 + Oloc1
// One CTA per chunk. A = [Phi1; Q'1] (tiles 0, 1 of the second half's image,
// bulk copy, K-major over key channels); B = Phi0 (tile 0 of the first half's
// image read through the transposed view), then Psi0 staged by the threads.
// ---------------------------------------------------------------------------
template <int DK, int DV, int NS>
__global__ void __launch_bounds__(128, 1) compose_kernel(ChunkParams p) {
  extern __shared__ __align__(128) uint8_t sm[];
  __shared__ uint64_t bar, bar_cp;
  __shared__ uint32_t tslot;
  const int Cs = p.Cs;  // 128
  const int tid = threadIdx.x, warp = tid >> 5;
  const MapGeom g1 = map_geom(DK, Cs), g2 = map_geom(DK, 2 * Cs);
  const uint32_t base = smem_u32(sm);
  const uint32_t bbase = base + 2 * g1.tile;
  if (tid == 0) mbar_init(&bar_cp, 1);
  TcCta cta;
  cta.init(&tslot, &bar, 512);
  const int64_t u0 = 2 * (int64_t)blockIdx.x, u1 = u0 + 1;
  const uint8_t* img0 = p.ma + u0 * g1.unit;
  const uint8_t* img1 = p.ma + u1 * g1.unit;
  if (tid == 0) {
    mbar_expect_tx(&bar_cp, 3 * g1.tile);
    bulk_g2s_big(base, img1, 2 * g1.tile, &bar_cp);
    bulk_g2s_big(bbase, img0, g1.tile, &bar_cp);
  }
  MmaSync drv{&bar, 0u, true};
  drv.ok = __syncthreads_and(mbar_wait(&bar_cp, 0) ? 1 : 0) != 0;
  const uint32_t lane = tmem_lane_base(warp);
  auto At = [&](int j) { return Tile{base + j * g1.tile, base + j * g1.tile + g1.half, 128u, DK * 16u}; };
  const Tile Bphi{bbase, bbase + g1.half, DK * 16u, 128u};  // Phi0: K = row, N = column
  if (drv.ok)
    drv.run([&] {
      for (int j = 0; j < 2; ++j)
        mma_tiles(cta.tmem + j * 128, At(j), Bphi, DK / 16, idesc_bf16(128, DK, 0, 1), NS, false);
    });
  const Tile Bpsi{bbase, bbase + DK * DV * 2u, 128u, DK * 16u};  // Psi0: K = row, N = column
  const float* psi0 = p.psi + u0 * DK * DV;
#pragma unroll 4
  for (int x = tid; x < DK * (DV / 8); x += 128) {
    int r, c8;
    piece_of<DV / 8>(x, r, c8);
    float v[8];
    ld8f(psi0 + slab_off(c8, r, DK), v);
    put_mn(Bpsi, r, c8, v);
  }
  if (drv.ok)
    drv.run([&] {
      for (int j = 0; j < 2; ++j)
        mma_tiles(cta.tmem + 256 + j * 128, At(j), Bpsi, DK / 16, idesc_bf16(128, DV, 0, 1), NS, false);
    });
  uint8_t* ma = p.ma2 + (int64_t)blockIdx.x * g2.unit;
  float* psi = p.psi2 + (int64_t)blockIdx.x * DK * DV;
  float* ol = p.ol2 + (int64_t)blockIdx.x * 2 * Cs * DV;
  const float* psi1 = p.psi + u1 * DK * DV;
  const float* ol1 = p.ol + u1 * Cs * DV;
  // tile 0 rows: Phi1 Phi0 (-> Phi), Phi1 Psi0 + Psi1 (-> Psi); tile 1 rows: Q'1 Phi0, Q'1 Psi0 + Oloc1
  for (int j = 0; j < 2; ++j) {
    const bool on = (j == 0 ? tid < DK : true) && drv.ok;
    for (int c = 0; c < DK; c += 16) {
      float v[16];
      tmem_ld16(cta.tmem + lane + j * 128 + c, v);
      if (on) {
        float a8[8], b8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) { a8[e] = v[e]; b8[e] = v[8 + e]; }
        if (j == 0) { map_put_phi(ma, g2, DK, tid, c, a8); map_put_phi(ma, g2, DK, tid, c + 8, b8); }
        else { map_put_q(ma, g2, DK, Cs + tid, c, a8); map_put_q(ma, g2, DK, Cs + tid, c + 8, b8); }
      }
    }
    for (int c = 0; c < DV; c += 16) {
      float v[16];
      tmem_ld16(cta.tmem + lane + 256 + j * 128 + c, v);
      if (on) {
        const float* a = j == 0 ? psi1 + slab_off(c, tid, DK) : ol1 + (int64_t)tid * DV + c;
        float* o = j == 0 ? psi + slab_off(c, tid, DK) : ol + (int64_t)(Cs + tid) * DV + c;
#pragma unroll
        for (int e = 0; e < 16; e += 4)
          *reinterpret_cast<float4*>(o + e) = make_float4(v[e] + a[e], v[e + 1] + a[e + 1], v[e + 2] + a[e + 2],
                                                          v[e + 3] + a[e + 3]);
      }
    }
  }
  // first half: Q'0 (tile 1 of h0 -> tile 1 of the chunk) and Oloc0 unchanged
  if (drv.ok) {
    const uint4* src = reinterpret_cast<const uint4*>(img0 + g1.tile);
    uint4* dst = reinterpret_cast<uint4*>(ma + g2.tile);
#pragma unroll 4
    for (int x = tid; x < (int)(g1.tile / 16); x += 128) dst[x] = src[x];
    const float4* s4 = reinterpret_cast<const float4*>(p.ol + u0 * Cs * DV);
    float4* d4 = reinterpret_cast<float4*>(ol);
#pragma unroll 4
    for (int x = tid; x < Cs * DV / 4; x += 128) d4[x] = s4[x];
  }
  cta.finish();
}

// ---------------------------------------------------------------------------
// scan_kernel: the only sequential step. One CTA per (batch, head, 32-column
// slab of the state) walks the chunks in order:
//   S_chunks[n] = S;   S <- Phi_n S + Psi_n
// The state slab stays on chip (registers, and bf16 hi/lo as the MMA's B
// operand). Phi_n (one tile) and the Psi_n slab arrive by bulk copies into two
// alternating buffers, issued two chunks ahead. The outputs, which need only
// the chunk-start states, are formed afterwards by out_kernel in parallel.
// ---------------------------------------------------------------------------
template <int DK, int NS>
__global__ void __launch_bounds__(128, 1) scan_kernel(ChunkParams p, const uint8_t* ma, const float* psi, int units,
                                                      int ulen) {
  extern __shared__ __align__(128) uint8_t sm[];
  __shared__ uint64_t bar, bar_c[2];
  __shared__ uint32_t tslot;
  constexpr int NW = kSlab;
  const int dv = p.dv, slabs = dv / NW;
  const int slab = blockIdx.x % slabs;
  const int bh = blockIdx.x / slabs;
  const int h = bh % p.H, b = bh / p.H;
  const int tid = threadIdx.x, warp = tid >> 5;
  const MapGeom g = map_geom(DK, ulen);
  const uint32_t PS = DK * NW * 4u;  // Psi slab bytes
  const uint32_t base = smem_u32(sm);
  const uint32_t psi_off = 2 * g.tile;
  const uint32_t s_off = psi_off + 2 * PS;
  const Tile Sb{base + s_off, base + s_off + NW * DK * 2u, 128u, DK * 16u};  // B: K = key row, N = column
  if (tid == 0) {
    mbar_init(&bar_c[0], 1);
    mbar_init(&bar_c[1], 1);
  }
  TcCta cta;
  cta.init(&tslot, &bar, 32);
  MmaSync drv{&bar, 0u, true};
  const uint32_t lane = tmem_lane_base(warp);
  const float* psi_s = reinterpret_cast<const float*>(static_cast<const uint8_t*>(sm) + psi_off);
  auto uid_of = [&](int n) { return ((int64_t)b * p.H + h) * units + n; };
  auto issue = [&](int n, int buf) {
    if (tid == 0) {
      mbar_expect_tx(&bar_c[buf], g.tile + PS);
      bulk_g2s_big(base + buf * g.tile, ma + uid_of(n) * g.unit, g.tile, &bar_c[buf]);
      bulk_g2s_big(base + psi_off + buf * PS,
                   reinterpret_cast<const uint8_t*>(psi + (uid_of(n) * slabs + slab) * DK * NW), PS, &bar_c[buf]);
    }
  };
  float st[NW];
  {
    const float* s0 = p.S0 ? p.S0 + (((int64_t)b * p.H + h) * DK) * dv + slab * NW : nullptr;
#pragma unroll
    for (int j = 0; j < NW; ++j) st[j] = (s0 && tid < DK) ? s0[(int64_t)tid * dv + j] : 0.f;
  }
  issue(0, 0);
  if (units > 1) issue(1, 1);
  const uint32_t id = idesc_bf16(128, NW, 0, 1);
  for (int n = 0; n < units && drv.ok; ++n) {
    const int buf = n & 1;
    if (tid < DK) {
#pragma unroll
      for (int j = 0; j < NW; j += 8) {
        float v[8];
#pragma unroll
        for (int e2 = 0; e2 < 8; ++e2) v[e2] = st[j + e2];
        put_mn(Sb, tid, j, v);
      }
    }
    fence_async_smem();  // the state operand is visible to the tensor core after the barrier below
    tc_fence_before();
    const bool c_ok = mbar_wait(&bar_c[buf], (uint32_t)(n >> 1) & 1u);
    if (!__syncthreads_and(c_ok ? 1 : 0)) { drv.ok = false; break; }
    const Tile Phi{base + buf * g.tile, base + buf * g.tile + g.half, 128u, DK * 16u};
    drv.run_synced([&] { mma_tiles(cta.tmem, Phi, Sb, DK / 16, id, NS, false); },
                    [&] {  // the chunk-start state leaves while the tensor core works
                      if (tid < DK && p.S_chunks) {
                        float* o = p.S_chunks + ((uid_of(n) * DK) + tid) * dv + slab * NW;
#pragma unroll
                        for (int j = 0; j < NW; j += 8) stg256(o + j, *reinterpret_cast<const float(*)[8]>(&st[j]));
                      }
                    });
    if (!drv.ok) break;
    float v[NW];
    tmem_ld_slab(cta.tmem + lane, v);
    if (tid < DK) {
      const float* add = psi_s + buf * (PS / 4) + tid * NW;
#pragma unroll
      for (int j = 0; j < NW; j += 4) {
        const float4 a4 = *reinterpret_cast<const float4*>(add + j);
        st[j] = v[j] + a4.x; st[j + 1] = v[j + 1] + a4.y; st[j + 2] = v[j + 2] + a4.z; st[j + 3] = v[j + 3] + a4.w;
      }
    }
    __syncthreads();  // buffer `buf` (Phi, Psi) is free again
    if (n + 2 < units) issue(n + 2, buf);
  }
  if (p.S_T && tid < DK && drv.ok) {
    float* o = p.S_T + (((int64_t)b * p.H + h) * DK + tid) * dv + slab * NW;
#pragma unroll
    for (int j = 0; j < NW; j += 8) stg256(o + j, *reinterpret_cast<const float(*)[8]>(&st[j]));
  }
  if (p.S_end && tid < DK && drv.ok) {
    float* o = p.S_end + (((int64_t)b * p.H + h) * DK + tid) * dv + slab * NW;
#pragma unroll
    for (int j = 0; j < NW; j += 8) stg256(o + j, *reinterpret_cast<const float(*)[8]>(&st[j]));
  }
  cta.finish();
}

// ---------------------------------------------------------------------------
// segmap_kernel: the affine map of a whole sequence segment, S_end = Phi_seg S0
// + Psi_seg, as the composition of its chunk maps (the exchange step of a scan
// split along T across ranks: each rank composes its segment, the maps are
// gathered, and each rank starts from its predecessors' composed maps). The
// composition is the scan run on the augmented state X = [Phi_acc | Psi_acc]
// (dk x (dk + dv)): X <- Phi_n X + [0 | Psi_n] from X = [I | 0]. One CTA per
// (batch, head, 32-column slab of X), with the same double-buffered bulk copies
// of Phi_n (and of the Psi_n slab for the Psi columns) as scan_kernel.
// ---------------------------------------------------------------------------
template <int DK, int NS>
__global__ void __launch_bounds__(128, 1) segmap_kernel(ChunkParams p, const uint8_t* ma, const float* psi, int units,
                                                        int ulen, float* Phi_seg, float* Psi_seg) {
  extern __shared__ __align__(128) uint8_t sm[];
  __shared__ uint64_t bar, bar_c[2];
  __shared__ uint32_t tslot;
  constexpr int NW = kSlab;
  const int dv = p.dv, vslabs = dv / NW, slabs = DK / NW + vslabs;
  const int slab = blockIdx.x % slabs;
  const int bh = blockIdx.x / slabs;
  const bool phi_part = slab < DK / NW;
  const int vs = slab - DK / NW;  // Psi slab index (Psi columns)
  const int tid = threadIdx.x, warp = tid >> 5;
  const MapGeom g = map_geom(DK, ulen);
  const uint32_t PS = DK * NW * 4u;
  const uint32_t base = smem_u32(sm);
  const uint32_t psi_off = 2 * g.tile;
  const uint32_t s_off = psi_off + 2 * PS;
  const Tile Sb{base + s_off, base + s_off + NW * DK * 2u, 128u, DK * 16u};
  if (tid == 0) {
    mbar_init(&bar_c[0], 1);
    mbar_init(&bar_c[1], 1);
  }
  TcCta cta;
  cta.init(&tslot, &bar, 32);
  MmaSync drv{&bar, 0u, true};
  const uint32_t lane = tmem_lane_base(warp);
  const float* psi_s = reinterpret_cast<const float*>(static_cast<const uint8_t*>(sm) + psi_off);
  auto issue = [&](int n, int buf) {
    if (tid == 0) {
      const int64_t uid = (int64_t)bh * units + n;
      mbar_expect_tx(&bar_c[buf], g.tile + (phi_part ? 0u : PS));
      bulk_g2s_big(base + buf * g.tile, ma + uid * g.unit, g.tile, &bar_c[buf]);
      if (!phi_part)
        bulk_g2s_big(base + psi_off + buf * PS, reinterpret_cast<const uint8_t*>(psi + (uid * vslabs + vs) * DK * NW),
                     PS, &bar_c[buf]);
    }
  };
  float st[NW];
#pragma unroll
  for (int j = 0; j < NW; ++j) st[j] = (phi_part && tid == slab * NW + j) ? 1.f : 0.f;
  issue(0, 0);
  if (units > 1) issue(1, 1);
  const uint32_t id = idesc_bf16(128, NW, 0, 1);
  for (int n = 0; n < units && drv.ok; ++n) {
    const int buf = n & 1;
    if (tid < DK) {
#pragma unroll
      for (int j = 0; j < NW; j += 8) {
        float v[8];
#pragma unroll
        for (int e2 = 0; e2 < 8; ++e2) v[e2] = st[j + e2];
        put_mn(Sb, tid, j, v);
      }
    }
    const bool c_ok = mbar_wait(&bar_c[buf], (uint32_t)(n >> 1) & 1u);
    if (!__syncthreads_and(c_ok ? 1 : 0)) { drv.ok = false; break; }
    const Tile Phi{base + buf * g.tile, base + buf * g.tile + g.half, 128u, DK * 16u};
    drv.run([&] { mma_tiles(cta.tmem, Phi, Sb, DK / 16, id, NS, false); });
    if (!drv.ok) break;
    float v[NW];
    tmem_ld_slab(cta.tmem + lane, v);
    if (tid < DK) {
      if (phi_part) {
#pragma unroll
        for (int j = 0; j < NW; ++j) st[j] = v[j];
      } else {
        const float* add = psi_s + buf * (PS / 4) + tid * NW;
#pragma unroll
        for (int j = 0; j < NW; j += 4) {
          const float4 a4 = *reinterpret_cast<const float4*>(add + j);
          st[j] = v[j] + a4.x; st[j + 1] = v[j + 1] + a4.y; st[j + 2] = v[j + 2] + a4.z; st[j + 3] = v[j + 3] + a4.w;
        }
      }
    }
    __syncthreads();  // buffer `buf` is free again
    if (n + 2 < units) issue(n + 2, buf);
  }
  if (tid < DK && drv.ok) {
    float* o = phi_part ? Phi_seg + ((int64_t)bh * DK + tid) * DK + slab * NW
                        : Psi_seg + ((int64_t)bh * DK + tid) * dv + vs * NW;
#pragma unroll
    for (int j = 0; j < NW; j += 8) stg256(o + j, *reinterpret_cast<const float(*)[8]>(&st[j]));
  }
  cta.finish();
}

// The identity map of an empty segment: Phi = I, Psi = 0 ([nh][dk][dk], [nh][dk][dv]).
__global__ void identity_map_kernel(float* __restrict__ Phi, float* __restrict__ Psi, int64_t nh, int dk, int dv) {
  const int64_t np = nh * dk * dk, ns = nh * dk * dv;
  for (int64_t x = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; x < np + ns; x += (int64_t)gridDim.x * blockDim.x) {
    if (x < np) Phi[x] = ((x / dk) % dk) == (x % dk) ? 1.f : 0.f;
    else Psi[x - np] = 0.f;
  }
}

// apply_map_kernel: S_out = Phi S_in + Psi per (sequence, head), fp32 on the CUDA
// cores (S_in NULL: S_out = Psi). Thread = one output element; rows of Phi and
// columns of S_in are read through the cache.
__global__ void apply_map_kernel(const float* __restrict__ Phi, const float* __restrict__ Psi,
                                 const float* __restrict__ S_in, float* __restrict__ S_out, int64_t nh, int dk, int dv) {
  const int64_t total = nh * dk * dv;
  for (int64_t x = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; x < total; x += (int64_t)gridDim.x * blockDim.x) {
    const int64_t m = x / ((int64_t)dk * dv);
    const int i = (int)((x / dv) % dk), j = (int)(x % dv);
    float acc = __ldg(Psi + x);
    if (S_in) {
      const float* ph = Phi + (m * dk + i) * dk;
      const float* sc = S_in + m * dk * dv + j;
      for (int c = 0; c < dk; ++c) acc = fmaf(__ldg(ph + c), __ldg(sc + (int64_t)c * dv), acc);
    }
    S_out[x] = acc;
  }
}

// ---------------------------------------------------------------------------
// out_kernel: outputs of one chunk from its start state, all chunks in
// parallel:  y = z * (Q' S0 + Oloc).
// A = Q' tiles of the map image (bulk copy, K-major over key channels),
// B = S0 (MN-major: K = key channel, N = value column), bulk-copied raw and
// converted in place (stage_raw). 256 threads: TMEM row t = tid % 128, the two
// warpgroups take alternate 32-column chunks.
// ---------------------------------------------------------------------------
template <int DK, int DV, typename T, int NS>
__global__ void __launch_bounds__(256, NS == 1 ? 2 : 1) out_kernel(ChunkParams p, const uint8_t* ma, const float* ol,
                                                                   int units, int ulen) {
  extern __shared__ __align__(128) uint8_t sm[];
  __shared__ uint64_t bar, bar_cp, bar_s0;
  __shared__ uint32_t tslot;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int64_t uid = blockIdx.x;
  const int n = (int)(uid % units);
  const int bh = (int)(uid / units);
  const int h = bh % p.H, b = bh / p.H;
  const MapGeom g = map_geom(DK, ulen);
  const int nq = g.ntile - 1;
  const uint32_t base = smem_u32(sm);
  // one pass reads only the hi planes of Q', so only they are copied: with
  // chunk 128 the CTA then needs 96 KB and two share an SM
  const uint32_t qt = NS == 1 ? g.half : g.tile;  // shared bytes per Q' tile
  const uint32_t s_off = (uint32_t)nq * qt;
  const Tile Sb{base + s_off, base + s_off + DK * DV * 2u, 128u, DK * 16u};
  if (tid == 0) {
    mbar_init(&bar_cp, 1);
    mbar_init(&bar_s0, 1);
  }
  TcCta cta;
  cta.init(&tslot, &bar, tmem_cols_for(nq * DV));
  if (tid == 0) {
    mbar_expect_tx(&bar_cp, nq * qt);
    if (NS == 1) {
      for (int j = 0; j < nq; ++j) bulk_g2s_big(base + j * qt, ma + uid * g.unit + (1 + j) * g.tile, qt, &bar_cp);
    } else {
      bulk_g2s_big(base, ma + uid * g.unit + g.tile, nq * g.tile, &bar_cp);
    }
  }
  uint32_t ph_s0 = 0;
  const bool s0_ok = stage_raw<true>(Sb, p.S_chunks + uid * DK * DV, DK, DV, 1.f, &bar_s0, ph_s0);
  MmaSync drv{&bar, 0u, true};
  drv.ok = __syncthreads_and((mbar_wait(&bar_cp, 0) && s0_ok) ? 1 : 0) != 0;
  const uint32_t id = idesc_bf16(128, DV, 0, 1);
  if (drv.ok)
    drv.run([&] {
      for (int j = 0; j < nq; ++j) {
        const Tile Q{base + j * qt, base + j * qt + (NS == 1 ? 0u : g.half), 128u, DK * 16u};
        mma_tiles(cta.tmem + j * DV, Q, Sb, DK / 16, id, NS, false);
      }
    });
  // y = z * (Q' S0 + Oloc) by 32 x 32 row blocks (rows_fill, rows_store): Oloc and
  // z come in and y goes out in whole lines, through shared memory that is free
  // once the products have completed.
  const uint32_t lane = tmem_lane_base(warp);
  const int ln = tid & 31, row0 = 32 * (warp & 3), wg = tid >> 7;
  constexpr uint32_t FB = row_block_bytes<float>(), CB = FB + row_block_bytes<T>();  // Oloc (then y), z
  constexpr int NCK = (DV + 63) / 64;  // 32-column chunks per warp
  const uint32_t wb = base + (uint32_t)warp * NCK * CB;
  auto gen = [&](uint32_t x) { return sm + (x - base); };  // shared address -> generic pointer
  const float* olu = ol + uid * ulen * DV;
  const T* zp = static_cast<const T*>(p.z);
  const int64_t ts = (int64_t)p.H * DV;
  const int64_t y0 = toff(p, b, (int64_t)n * ulen, h, DV);  // token 0 of the unit
  for (int j = 0; j < nq; ++j) {
    const int nrj = ulen - j * 128 < 128 ? ulen - j * 128 : 128;  // rows of this 128-row tile
    const int64_t yj = y0 + (int64_t)j * 128 * ts;
    if (drv.ok) {
      int k = 0;
      for (int c = wg * 32; c < DV; c += 64, ++k) {
        rows_fill<float>(wb + k * CB, olu + (int64_t)j * 128 * DV, DV, row0, nrj, c);
        if (zp) rows_fill<T>(wb + k * CB + FB, zp + yj, ts, row0, nrj, c);
      }
    }
    cp_async_wait_all();
    __syncwarp();
    {
      int k = 0;
      for (int c = wg * 32; c < DV; c += 64, ++k) {
        float v[32];
        tmem_ld32(cta.tmem + lane + j * DV + c, v);
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8) {
          float a8[8], z8[8];
          row8_get<float>(gen(wb + k * CB), ln, q8, a8);
          if (zp) {
            row8_get<T>(gen(wb + k * CB + FB), ln, q8, z8);
          } else {  // y = o when z is absent
#pragma unroll
            for (int e2 = 0; e2 < 8; ++e2) z8[e2] = 1.f;
          }
#pragma unroll
          for (int e2 = 0; e2 < 8; ++e2) a8[e2] = (v[8 * q8 + e2] + a8[e2]) * z8[e2];
          row8_put(gen(wb + k * CB), ln, q8, a8);
        }
      }
    }
    __syncwarp();
    if (drv.ok) {
      int k = 0;
      for (int c = wg * 32; c < DV; c += 64, ++k) rows_store<T>(gen(wb + k * CB), static_cast<T*>(p.y) + yj, ts, row0, nrj, c);
    }
    __syncwarp();
  }
  cta.finish();
}

}  // namespace muir
