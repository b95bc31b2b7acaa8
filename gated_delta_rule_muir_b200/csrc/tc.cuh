// Blackwell (sm_100a) tensor-core primitives: tcgen05.mma with shared-memory
// operand descriptors, fp32 accumulators in tensor memory (TMEM), completion
// tracked through an mbarrier, and TMEM -> register loads.
//
// Operand tiles live in shared memory in the "no-swizzle" canonical layout made
// of 8 x 16-byte core matrices (8 rows of 8 bf16). A tile covering MN rows
// (multiple of 8) and KT contraction indices (multiple of 16) is stored as
// MN/8 groups, each group holding KT/8 core matrices back to back:
//
//   K-major tile  (row = MN index m, 8 consecutive k per 16-byte row):
//       byte(m, k) = (m/8)*SBO + (k/8)*128 + (m%8)*16 + (k%8)*2
//   MN-major tile (row = contraction index k, 8 consecutive m per 16-byte row):
//       byte(k, m) = (m/8)*SBO + (k/8)*128 + (k%8)*16 + (m%8)*2
//
// with SBO = KT*16 (distance between MN groups) and LBO = 128 (distance between
// core matrices adjacent along K). One MMA consumes K = 16 = two core matrices
// along K, so the k-th MMA step starts 256 bytes further. The same physical
// tile of a row-major matrix X[rows][cols] can be fed as a K-major operand
// (contract over cols) or as an MN-major operand (contract over rows).
//
// fp32 operands are split into bf16 hi + lo parts (x = hi + lo + O(2^-17 |x|));
// a product is accumulated as hi*hi + hi*lo + lo*hi, which keeps ~2^-16
// relative accuracy at bf16 tensor-core rate ("3-pass bf16").
#pragma once

#include "common.cuh"

namespace muir {

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---- mbarrier --------------------------------------------------------------

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Wait for the phase with the given parity to complete. Bounded: gives up once
// limit_ns of global time have passed since the first check, records the
// timeout in the device status word and returns false. Each try may suspend the
// thread in hardware for up to 20 us (it resumes as soon as the phase completes),
// so a waiting warp does not spin on the issue slots other warps need.
__device__ __forceinline__ bool mbar_wait_for(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  const uint32_t a = smem_u32(bar);
  uint64_t t0 = 0;
  for (uint32_t it = 0;; ++it) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, 20000;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(a), "r"(parity)
        : "memory");
    if (ok) return true;
    if ((it & 3) == 0) {
      const uint64_t now = globaltimer_ns();
      if (t0 == 0) t0 = now;
      else if (now - t0 > limit_ns) { flag_timeout(); return false; }
    }
  }
}

// The library's waits: about one second.
constexpr uint64_t kWaitLimitNs = 1000000000ull;
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  return mbar_wait_for(bar, parity, kWaitLimitNs);
}

// ---- bulk asynchronous copies (global -> shared, completion on an mbarrier) --

// Arrive on `bar` (count 1) and announce `bytes` of incoming bulk-copy traffic.
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

// Copy `bytes` (multiple of 16, both addresses 16-byte aligned) from global to
// shared memory; completes as transaction bytes on `bar`. No multicast.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint64_t* bar) {
  MUIR_SMEM_GUARD(dst, bytes);
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// Copy `bytes` (multiple of 16, both addresses 16-byte aligned) from shared to
// global memory, in this thread's bulk-async group. No multicast.
__device__ __forceinline__ void bulk_s2g(void* dst, uint32_t src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(src), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until this thread's committed bulk copies have completed.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// ---- fences ----------------------------------------------------------------

// Generic-proxy shared-memory writes -> visible to the tensor core (async proxy).
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// ---- TMEM allocation (whole warp) ------------------------------------------

__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// ---- descriptors -----------------------------------------------------------

// Instruction descriptor, kind::f16: bf16 A and B, fp32 accumulator, dense.
// a_mn / b_mn: 0 = K-major, 1 = MN-major.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int a_mn, int b_mn) {
  return (1u << 4)                        // D format: f32
         | (1u << 7)                      // A format: bf16
         | (1u << 10)                     // B format: bf16
         | (uint32_t(a_mn) << 15) | (uint32_t(b_mn) << 16) |
         (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

// Shared-memory matrix descriptor, no swizzle (layout type 0), sm_100 version bit.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)(lbo >> 4) << 16) | ((uint64_t)(sbo >> 4) << 32) |
         (1ull << 46);
}

// Shared-memory matrix descriptor with the 128-byte swizzle (layout type 2),
// sm_100 version bit; the tile base must be 1024-byte aligned. Rows are 128
// bytes (64 bf16), the 16-byte chunk c of row r stored at chunk c ^ (r % 8).
//   K-major operand (rows = M or N, columns = K): SBO = 1024 between 8-row
//     groups; the K step of 16 elements adds 32 bytes inside the row, and every
//     64 columns of K start a new box of rows.
//   MN-major operand (rows = K, columns = M or N): SBO = 1024 between 8-row
//     groups along K, LBO = the distance between 64-column boxes along M/N; the
//     K step of 16 rows adds 2048 bytes.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)(lbo >> 4) << 16) | ((uint64_t)(sbo >> 4) << 32) |
         (1ull << 46) | (2ull << 61);
}

// ---- MMA issue (single thread) ---------------------------------------------

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accum)
      : "memory");
}

// Arrive once on `bar` when all previously issued MMAs of this thread complete.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// A staged operand tile: bf16 hi and lo parts in shared memory, with the byte
// distance between core matrices adjacent along K (lbo) and along M/N (sbo).
// put_k / put_mn below write tiles whose natural view has lbo = 128. The same
// memory read with lbo and sbo swapped (transposed()) is the other major: a
// tile written by put_k as a K-major operand is, transposed, an MN-major
// operand of the transposed matrix, and vice versa.
struct Tile {
  uint32_t hi, lo;  // shared addresses (16-byte aligned)
  uint32_t lbo;     // K-direction core-matrix stride
  uint32_t sbo;     // MN-direction core-matrix stride
};

__device__ __forceinline__ Tile transposed(const Tile& t) { return Tile{t.hi, t.lo, t.sbo, t.lbo}; }

// A staged operand in 128-byte-swizzled rows: bf16 hi and lo planes (each
// 1024-byte aligned), row r of the matrix in 64-column boxes `box` bytes apart.
// Written row by row (put_sw), it is read as the K-major operand (rows = M or
// N) or the MN-major one (rows = K): a sweep whose 8 threads per shared-memory
// phase store 8 consecutive 16-byte pieces of one row lands them in 8 distinct
// bank groups.
struct SwTile {
  uint32_t hi, lo;
  uint32_t box;
};

// Operand views for the MMA loop below: each gives the shared-memory descriptor
// of its hi or lo plane at MMA step j (K = 16 per step).
//   NoSw: a no-swizzle Tile as stored (its lbo is the K-direction stride).
//   SwK:  a SwTile read K-major (rows = M or N, columns = K).
//   SwMN: a SwTile read MN-major (rows = K, columns = M or N).
struct NoSw {
  Tile t;
  __device__ __forceinline__ uint64_t desc(int j, bool lo) const {
    return sdesc((lo ? t.lo : t.hi) + (uint32_t)j * 2u * t.lbo, t.lbo, t.sbo);
  }
};
struct SwK {
  SwTile t;
  __device__ __forceinline__ uint64_t desc(int j, bool lo) const {
    return sdesc_sw128((lo ? t.lo : t.hi) + (uint32_t)(j >> 2) * t.box + (uint32_t)(j & 3) * 32u, 16u, 1024u);
  }
};
struct SwMN {
  SwTile t;
  __device__ __forceinline__ uint64_t desc(int j, bool lo) const {
    return sdesc_sw128((lo ? t.lo : t.hi) + (uint32_t)j * 2048u, t.box, 1024u);
  }
};

// D[tmem] (+)= A * B over `ksteps` MMA steps of K = 16. M = 128 rows of A
// (lanes of D), N columns of B. nsplit = 1 (hi*hi), 3 (hi*hi + hi*lo + lo*hi),
// or 2 (hi*hi + A.lo*B.hi, for a B exact in bf16).
template <typename OA, typename OB>
__device__ __forceinline__ void mma_ops(uint32_t d_tmem, const OA& A, const OB& B, int ksteps, uint32_t idesc,
                                        int nsplit, bool accumulate) {
  for (int j = 0; j < ksteps; ++j) {
    const uint64_t ah = A.desc(j, false), bh = B.desc(j, false);
    mma_bf16(d_tmem, ah, bh, idesc, (accumulate || j > 0) ? 1u : 0u);
    if (nsplit == 3) {
      mma_bf16(d_tmem, ah, B.desc(j, true), idesc, 1u);
      mma_bf16(d_tmem, A.desc(j, true), bh, idesc, 1u);
    } else if (nsplit == 2) {
      mma_bf16(d_tmem, A.desc(j, true), bh, idesc, 1u);
    }
  }
}

// A K-major operand tile over COLS columns (rows = M or N, at most 128; hi and
// lo planes `plane` bytes apart, base 1024-byte aligned): 128-byte-swizzled rows
// when COLS is a multiple of 64, the no-swizzle layout otherwise (rows of 64
// bytes cannot take the 128-byte swizzle). kview gives its K-major MMA view.
template <int COLS>
__device__ __forceinline__ auto kmajor_tile(uint32_t a, uint32_t plane) {
  if constexpr (COLS % 64 == 0) return SwTile{a, a + plane, 128u * 128u};
  else return Tile{a, a + plane, 128u, (uint32_t)COLS * 16u};
}
__device__ __forceinline__ SwK kview(const SwTile& t) { return SwK{t}; }
__device__ __forceinline__ NoSw kview(const Tile& t) { return NoSw{t}; }

// The no-swizzle pair, the common case.
__device__ __forceinline__ void mma_tiles(uint32_t d_tmem, const Tile& A, const Tile& B, int ksteps, uint32_t idesc,
                                          int nsplit, bool accumulate) {
  mma_ops(d_tmem, NoSw{A}, NoSw{B}, ksteps, idesc, nsplit, accumulate);
}

// ---- operand staging (any thread) ------------------------------------------

__device__ __forceinline__ void split8(const float (&x)[8], uint4& hi, uint4& lo) {
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&hi);
  __nv_bfloat162* l = reinterpret_cast<__nv_bfloat162*>(&lo);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __nv_bfloat162 hh = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
    const float2 hf = __bfloat1622float2(hh);
    h[i] = hh;
    l[i] = __floats2bfloat162_rn(x[2 * i] - hf.x, x[2 * i + 1] - hf.y);
  }
}

// 16-byte store to a shared-memory address. A plain C++ store through the
// generic alias of the address: the compiler sees a shared-memory store and can
// keep issuing the next staging iteration's global loads ahead of it (an asm
// store with a memory clobber would serialise every staging loop). Ordering
// with the tensor core is established by fence_async_smem() + a CTA barrier.
__device__ __forceinline__ void sts128(uint32_t addr, const uint4& v) {
  MUIR_SMEM_GUARD(addr, 16u);
  *reinterpret_cast<uint4*>(__cvta_shared_to_generic(addr)) = v;
}

// Row r, columns c8..c8+7 of a SwTile.
__device__ __forceinline__ void put_sw(const SwTile& t, int r, int c8, const float (&x)[8]) {
  uint4 hi, lo;
  split8(x, hi, lo);
  const uint32_t off = (uint32_t)(c8 >> 6) * t.box + (uint32_t)r * 128u + ((uint32_t)(((c8 >> 3) & 7) ^ (r & 7)) << 4);
  sts128(t.hi + off, hi);
  sts128(t.lo + off, lo);
}

// K-major (natural view, lbo = 128): 8 consecutive contraction indices k8..k8+7 of MN row m.
__device__ __forceinline__ void put_k(const Tile& t, int m, int k8, const float (&x)[8]) {
  uint4 hi, lo;
  split8(x, hi, lo);
  const uint32_t off = (uint32_t)(m >> 3) * t.sbo + (uint32_t)(k8 >> 3) * 128u + (uint32_t)(m & 7) * 16u;
  sts128(t.hi + off, hi);
  sts128(t.lo + off, lo);
}

// Row r (the K-major view's M or N index), columns c8..c8+7 of either kind of tile.
__device__ __forceinline__ void put_op(const Tile& t, int r, int c8, const float (&x)[8]) { put_k(t, r, c8, x); }
__device__ __forceinline__ void put_op(const SwTile& t, int r, int c8, const float (&x)[8]) { put_sw(t, r, c8, x); }

// Staging sweeps over a rows x (8 G) matrix in 8-element pieces (G a power of
// two, rows a multiple of 8). put_k and put_mn store a piece to the bank group
// given by its row & 7, and a 128-bit shared-memory access serves a warp in four
// phases of 8 consecutive threads, so piece x goes to row ((x / 8G) * 8 + x % 8),
// column block (x / 8) % G: the 8 threads of a phase take 8 consecutive rows of
// one column block and store without bank conflicts (taking one row's 8 column
// blocks would put all 8 in one bank group). In global memory a warp then reads
// 8 rows x 4 pieces, the same number of sectors as 2 rows x 16 pieces.
template <int G>
__device__ __forceinline__ void piece_of(int x, int& r, int& c8) {
  static_assert(G > 0 && (G & (G - 1)) == 0, "G must be a power of two");
  constexpr int lg = G == 1 ? 0 : G == 2 ? 1 : G == 4 ? 2 : G == 8 ? 3 : G == 16 ? 4 : G == 32 ? 5 : 6;
  static_assert((1 << lg) == G, "G out of range");
  r = ((x >> (3 + lg)) << 3) | (x & 7);
  c8 = ((x >> 3) & (G - 1)) << 3;
}
// Piece order for a sweep reading rows of element type T from global memory:
// piece_of for fp32 rows (a warp reads 8 rows x 128 bytes, whole lines); for
// bf16 rows plain row-major order (a warp reads 2 rows x 256 bytes) keeps the
// loads in whole lines, at the price of bank conflicts on the stores.
template <typename T, int G>
__device__ __forceinline__ void row_piece(int x, int& r, int& c8) {
  if constexpr (sizeof(T) == 4) {
    piece_of<G>(x, r, c8);
  } else {
    r = x / G;
    c8 = (x % G) * 8;
  }
}

// The same for a G known only at run time (a power of two).
__device__ __forceinline__ void piece_of_rt(int x, int G, int& r, int& c8) {
  const int lg = 31 - __clz(G);
  r = ((x >> (3 + lg)) << 3) | (x & 7);
  c8 = ((x >> 3) & (G - 1)) << 3;
}
// For a source read back from row-major shared memory: the column block is also
// rotated by the row within the phase, so that the phase's reads spread over
// the bank groups as well.
__device__ __forceinline__ void piece_of_rot(int x, int G, int& r, int& c8) {
  const int lg = 31 - __clz(G);
  r = ((x >> (3 + lg)) << 3) | (x & 7);
  c8 = (((x >> 3) + (x & 7)) & (G - 1)) << 3;
}
// The same for a SwTile destination (G >= 8): row i of the phase takes column
// block c ^ (i / 2). The reads then fall on the four 32-byte positions of a
// 128-byte line twice each, as with the rotation, and the swizzled stores (chunk
// (c ^ (i / 2)) ^ i for rows i = 0..7) hit 8 distinct bank groups; the rotation
// would put all 8 of them in one.
__device__ __forceinline__ void piece_of_swz(int x, int G, int& r, int& c8) {
  const int lg = 31 - __clz(G);
  r = ((x >> (3 + lg)) << 3) | (x & 7);
  c8 = (((x >> 3) & (G - 1)) ^ ((x & 7) >> 1)) << 3;
}

// 8 values that are exact in bf16, already packed (uint4 of 8 bf16): the hi
// plane only (their lo part is zero and is never read: 1-pass, or 2-pass with
// this tile as the exact B operand). K-major and MN-major offsets as put_k / put_mn.
__device__ __forceinline__ void put_k_raw(const Tile& t, int m, int k8, const uint4& v) {
  sts128(t.hi + (uint32_t)(m >> 3) * t.sbo + (uint32_t)(k8 >> 3) * 128u + (uint32_t)(m & 7) * 16u, v);
}
__device__ __forceinline__ void put_mn_raw(const Tile& t, int k, int m8, const uint4& v) {
  sts128(t.hi + (uint32_t)(m8 >> 3) * t.sbo + (uint32_t)(k >> 3) * 128u + (uint32_t)(k & 7) * 16u, v);
}

// MN-major (natural view, lbo = 128): 8 consecutive MN indices m8..m8+7 of contraction row k.
__device__ __forceinline__ void put_mn(const Tile& t, int k, int m8, const float (&x)[8]) {
  uint4 hi, lo;
  split8(x, hi, lo);
  const uint32_t off = (uint32_t)(m8 >> 3) * t.sbo + (uint32_t)(k >> 3) * 128u + (uint32_t)(k & 7) * 16u;
  sts128(t.hi + off, hi);
  sts128(t.lo + off, lo);
}

// Global-memory image of staged tiles: the same byte layout as put_k, written to
// global memory so that a consumer can bring it into shared memory with one bulk
// copy. `hi` points at the hi block, the lo block follows `lo_off` bytes later.
__device__ __forceinline__ void gput_k(uint8_t* hi, uint32_t lo_off, uint32_t sbo, int m, int k8, const float (&x)[8]) {
  uint4 h, l;
  split8(x, h, l);
  const uint32_t off = (uint32_t)(m >> 3) * sbo + (uint32_t)(k8 >> 3) * 128u + (uint32_t)(m & 7) * 16u;
  *reinterpret_cast<uint4*>(hi + off) = h;
  *reinterpret_cast<uint4*>(hi + lo_off + off) = l;
}

// 4 consecutive columns (c4 % 4 == 0) of row m into a global tile image.
__device__ __forceinline__ void gput_k4(uint8_t* hi, uint32_t lo_off, uint32_t sbo, int m, int c4, const float (&x)[4]) {
  uint2 h, l;
  __nv_bfloat162* hh = reinterpret_cast<__nv_bfloat162*>(&h);
  __nv_bfloat162* ll = reinterpret_cast<__nv_bfloat162*>(&l);
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const __nv_bfloat162 b = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
    const float2 f = __bfloat1622float2(b);
    hh[i] = b;
    ll[i] = __floats2bfloat162_rn(x[2 * i] - f.x, x[2 * i + 1] - f.y);
  }
  const uint32_t off = (uint32_t)(m >> 3) * sbo + (uint32_t)(c4 >> 3) * 128u + (uint32_t)(m & 7) * 16u + (uint32_t)(c4 & 7) * 2u;
  *reinterpret_cast<uint2*>(hi + off) = h;
  *reinterpret_cast<uint2*>(hi + lo_off + off) = l;
}

// ---- TMEM -> registers -----------------------------------------------------

// Lane base of warp w's TMEM sub-partition.
__device__ __forceinline__ uint32_t tmem_lane_base(int warp) { return (uint32_t)((warp & 3) * 32) << 16; }

// 16 consecutive fp32 columns of this thread's lane (row), completes before return.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// 8 consecutive fp32 columns.
// 32 consecutive fp32 columns of this thread's lane (one load, one wait).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&v)[8]) {
  uint32_t r[8];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}

template <int N>
__device__ __forceinline__ void tmem_ld_slab(uint32_t taddr, float (&v)[N]) {
  static_assert(N == 16 || N == 32, "slab width");
  if constexpr (N == 32) tmem_ld32(taddr, v);
  else tmem_ld16(taddr, v);
}

// ---- a tiny synchronous MMA driver ----------------------------------------
//
// Holds the mbarrier phase. Usage (all threads of a 128-thread CTA):
//   stage operands; drv.run([&]{ mma_tiles(...); ... });   // waits for completion
struct MmaSync {
  uint64_t* bar;
  uint32_t phase;
  bool ok;

  // All threads: publish staged smem to the tensor core, let thread 0 issue the
  // MMAs given by `issue`, commit, and wait for completion. Returns false (and
  // leaves `ok` false) if the bounded wait expired.
  template <typename F>
  __device__ __forceinline__ bool run(F issue) {
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0) {
      tc_fence_after();
      issue();
      mma_commit(bar);
    }
    const bool done = __syncthreads_and(mbar_wait(bar, phase) ? 1 : 0) != 0;
    phase ^= 1u;
    tc_fence_after();
    ok = ok && done;
    return done;
  }

  // As run_overlap, for callers that have already made their operand writes
  // visible (fence_async_smem + tc_fence_before by every thread, then a CTA
  // barrier): saves that barrier.
  template <typename F, typename W>
  __device__ __forceinline__ bool run_synced(F issue, W work) {
    if (threadIdx.x == 0) {
      tc_fence_after();
      issue();
      mma_commit(bar);
    }
    work();
    const bool done = __syncthreads_and(mbar_wait(bar, phase) ? 1 : 0) != 0;
    phase ^= 1u;
    tc_fence_after();
    ok = ok && done;
    return done;
  }

  // Same, but all threads run `work` (which must not touch the staged operands
  // or the accumulators of these MMAs) while the tensor core executes.
  template <typename F, typename W>
  __device__ __forceinline__ bool run_overlap(F issue, W work) {
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0) {
      tc_fence_after();
      issue();
      mma_commit(bar);
    }
    work();
    const bool done = __syncthreads_and(mbar_wait(bar, phase) ? 1 : 0) != 0;
    phase ^= 1u;
    tc_fence_after();
    ok = ok && done;
    return done;
  }
};

}  // namespace muir
