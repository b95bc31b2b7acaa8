// Shared device helpers: element loads/stores for the two input dtypes, and the
// library's device status word (set when a bounded wait runs out).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <type_traits>

namespace muir {

// Device-side status word: bit 0 = a bounded wait expired. Read and cleared by
// muir_device_status(). One word per device context of the library.
__device__ unsigned int g_status;

constexpr unsigned int kStatusTimeout = 1u;
// a checking build found an index out of its bounds: a shared-memory address, a
// (batch, token, head) index of an input or output tensor, a Gram image index
constexpr unsigned int kStatusBoundsSmem = 2u, kStatusBoundsToken = 4u, kStatusBoundsImage = 8u;
constexpr unsigned int kStatusBounds = kStatusBoundsSmem | kStatusBoundsToken | kStatusBoundsImage;

__device__ __forceinline__ void flag_timeout() { atomicOr(&g_status, kStatusTimeout); }

// Checking builds (-DMUIR_CHECK): the central access helpers test their indices,
// and a failed test records kStatusBounds in the status word and skips (or
// redirects to an in-bounds address) the access instead of trapping. Without
// MUIR_CHECK the tests compile away.
#ifdef MUIR_CHECK
__device__ __forceinline__ bool check_bounds(bool ok, unsigned int what) {
  if (!ok) atomicOr(&g_status, what);
  return ok;
}
// Upper end of this CTA's shared-memory window, with 1 KB of slack for the
// region the system reserves ahead of the kernel's own shared memory.
__device__ __forceinline__ uint32_t smem_window_end() {
  uint32_t n;
  asm("mov.u32 %0, %%total_smem_size;" : "=r"(n));
  return n + 1024u;
}
#define MUIR_SMEM_GUARD(addr, bytes) \
  if (!::muir::check_bounds((uint32_t)(addr) + (uint32_t)(bytes) <= ::muir::smem_window_end(), \
                            ::muir::kStatusBoundsSmem))                                          \
  return
#else
#define MUIR_SMEM_GUARD(addr, bytes)
#endif

// ---- element access -----------------------------------------------------

template <typename T> struct Elt;

template <> struct Elt<float> {
  static __device__ __forceinline__ float ld(const float* p) { return __ldg(p); }
  static __device__ __forceinline__ float ld_or_one(const float* p) { return p ? __ldg(p) : 1.f; }
  // 8 consecutive elements through a generic pointer (e.g. shared memory).
  static __device__ __forceinline__ void ld8g(const float* p, float (&o)[8]) {
    const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
    o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w;
    o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
  }
  static __device__ __forceinline__ void st(float* p, float x) { *p = x; }
  // 8 consecutive elements (p 32-byte aligned).
  static __device__ __forceinline__ void ld8(const float* p, float (&o)[8]) {
    float4 a = __ldg(reinterpret_cast<const float4*>(p));
    float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w;
    o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
  }
  static __device__ __forceinline__ void ld4(const float* p, float (&o)[4]) {
    float4 a = __ldg(reinterpret_cast<const float4*>(p));
    o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w;
  }
  static __device__ __forceinline__ void st4(float* p, const float (&o)[4]) {
    *reinterpret_cast<float4*>(p) = make_float4(o[0], o[1], o[2], o[3]);
  }
  static __device__ __forceinline__ void st8(float* p, const float (&o)[8]) {
    reinterpret_cast<float4*>(p)[0] = make_float4(o[0], o[1], o[2], o[3]);
    reinterpret_cast<float4*>(p)[1] = make_float4(o[4], o[5], o[6], o[7]);
  }
};

template <> struct Elt<__nv_bfloat16> {
  using T = __nv_bfloat16;
  static __device__ __forceinline__ float ld(const T* p) { return __bfloat162float(__ldg(p)); }
  static __device__ __forceinline__ float ld_or_one(const T* p) { return p ? __bfloat162float(__ldg(p)) : 1.f; }
  static __device__ __forceinline__ void ld8g(const T* p, float (&o)[8]) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(h[i]);
      o[2 * i] = f.x; o[2 * i + 1] = f.y;
    }
  }
  static __device__ __forceinline__ void st(T* p, float x) { *p = __float2bfloat16_rn(x); }
  static __device__ __forceinline__ void ld8(const T* p, float (&o)[8]) {
    uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 f = __bfloat1622float2(h[i]);
      o[2 * i] = f.x; o[2 * i + 1] = f.y;
    }
  }
  static __device__ __forceinline__ void ld4(const T* p, float (&o)[4]) {
    uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
    float2 a = __bfloat1622float2(h[0]), b = __bfloat1622float2(h[1]);
    o[0] = a.x; o[1] = a.y; o[2] = b.x; o[3] = b.y;
  }
  static __device__ __forceinline__ void st4(T* p, const float (&o)[4]) {
    uint2 u;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
    h[0] = __floats2bfloat162_rn(o[0], o[1]);
    h[1] = __floats2bfloat162_rn(o[2], o[3]);
    *reinterpret_cast<uint2*>(p) = u;
  }
  static __device__ __forceinline__ void st8(T* p, const float (&o)[8]) {
    uint4 u;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(o[2 * i], o[2 * i + 1]);
    *reinterpret_cast<uint4*>(p) = u;
  }
};

// 8 consecutive elements held in their storage type until used (for bf16 half the
// registers of 8 floats), so that many loads can be in flight at once.
template <typename T> struct Pack8;
template <> struct Pack8<float> {
  float4 a, b;
  __device__ __forceinline__ void ld(const float* p) {
    a = __ldg(reinterpret_cast<const float4*>(p));
    b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  }
  __device__ __forceinline__ void set_one() { a = b = make_float4(1.f, 1.f, 1.f, 1.f); }
  // load, or all ones when p is null (an absent gate)
  __device__ __forceinline__ void ld_or_one(const float* p) { if (p) ld(p); else set_one(); }
  __device__ __forceinline__ void get(float (&o)[8]) const {
    o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w;
    o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
  }
};
template <> struct Pack8<__nv_bfloat16> {
  uint4 u;
  __device__ __forceinline__ void ld(const __nv_bfloat16* p) { u = __ldg(reinterpret_cast<const uint4*>(p)); }
  __device__ __forceinline__ void set_one() { u = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u); }
  __device__ __forceinline__ void ld_or_one(const __nv_bfloat16* p) { if (p) ld(p); else set_one(); }
  __device__ __forceinline__ void get(float (&o)[8]) const {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(h[i]);
      o[2 * i] = f.x; o[2 * i + 1] = f.y;
    }
  }
};

// 8 floats to global memory: one 32-byte store where p is 32-byte aligned, two
// 16-byte stores where it is only 16-byte aligned (the C ABI requires 16 bytes
// of its callers' pointers, and a 32-byte vector store to an address that is
// not 32-byte aligned is a fault).
__device__ __forceinline__ void stg256(float* p, const float (&v)[8]) {
  if ((reinterpret_cast<uintptr_t>(p) & 31u) == 0) {
    asm volatile("st.global.v8.f32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "f"(v[0]), "f"(v[1]), "f"(v[2]),
                 "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7])
                 : "memory");
  } else {
    reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
  }
}

// 16 floats (p 16-byte aligned) in two 32-byte stores (see stg256).
__device__ __forceinline__ void stg_row16(float* p, const float (&v)[16]) {
  float a[8], b[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) { a[j] = v[j]; b[j] = v[8 + j]; }
  stg256(p, a);
  stg256(p + 8, b);
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

}  // namespace muir
