// libmuir.so: the C ABI declared in include/muir.h. Validates arguments, sizes
// workspaces and launches the kernels; all arithmetic of the operator happens
// in the kernels included below.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/muir.h"
#include "../../include/muir_profile.h"
#include "common.cuh"
#include "decode.cuh"
#include "selftest.cuh"
#include "chunk.cuh"
#include "gram.cuh"
#include "chunk_bwd.cuh"
#include "gate_proj.cuh"
#include "gate_proj_tma.cuh"

namespace {

thread_local std::string g_err;

int fail(int code, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_err = buf;
  return code;
}

int cuda_check(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(MUIR_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return MUIR_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ---- launch accounting and optional per-launch event timing ---------------
struct ProfRec {
  const char* phase;
  const char* name;
  cudaEvent_t a, b;
};
thread_local const char* g_phase = "";  // "fwd" / "bwd" while inside a chunk entry point
struct Prof {
  bool on = false;
  std::vector<ProfRec> recs;
  std::vector<cudaEvent_t> pool;
  int64_t launches = 0;
  cudaEvent_t get() {
    if (!pool.empty()) {
      cudaEvent_t e = pool.back();
      pool.pop_back();
      return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
  }
};
Prof g_prof;

// Brackets one kernel launch on stream s (construct right before the launch).
struct Launch {
  cudaStream_t s;
  const char* name;
  cudaEvent_t b = nullptr;
  ProfRec* rec = nullptr;
  Launch(const char* n, cudaStream_t st) : s(st), name(n) {
    ++g_prof.launches;
    if (g_prof.on) {
      ProfRec r{g_phase, n, g_prof.get(), g_prof.get()};
      cudaEventRecord(r.a, s);
      g_prof.recs.push_back(r);
      b = r.b;
    }
  }
  ~Launch() {
    if (b) cudaEventRecord(b, s);
  }
};
bool dim_ok(int d) { return d == 32 || d == 64 || d == 128; }

}  // namespace

extern "C" {

int muir_version(void) { return 103; }

const char* muir_last_error(void) { return g_err.c_str(); }

int muir_device_status(void* stream) {
  g_err.clear();
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return cuda_check("cudaStreamSynchronize");
  unsigned int host = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&host, muir::g_status, sizeof host) != cudaSuccess) return cuda_check("read status");
  if (cudaMemcpyToSymbol(muir::g_status, &zero, sizeof zero) != cudaSuccess) return cuda_check("clear status");
  if (host & muir::kStatusTimeout) return fail(MUIR_ERR_TIMEOUT, "a bounded device wait expired");
  if (host & muir::kStatusBounds)
    return fail(MUIR_ERR_BOUNDS, "an index failed its bounds check (checking build):%s%s%s",
                (host & muir::kStatusBoundsSmem) ? " shared-memory address" : "",
                (host & muir::kStatusBoundsToken) ? " tensor (batch, token, head) index" : "",
                (host & muir::kStatusBoundsImage) ? " Gram image index" : "");
  return MUIR_OK;
}

int muir_state_init(float* S, const float* S_src, int64_t n_seq, int32_t H, int32_t dk, int32_t dv, void* stream) {
  g_err.clear();
  if (!S) return fail(MUIR_ERR_INVALID_ARG, "state_init: S is NULL");
  if (n_seq < 0 || H <= 0 || !dim_ok(dk) || !dim_ok(dv))
    return fail(MUIR_ERR_UNSUPPORTED, "state_init: unsupported sizes n_seq=%lld H=%d dk=%d dv=%d", (long long)n_seq, H,
                dk, dv);
  if (!aligned16(S) || (S_src && !aligned16(S_src))) return fail(MUIR_ERR_INVALID_ARG, "state_init: misaligned pointer");
  const int64_t n4 = n_seq * H * (int64_t)dk * dv / 4;
  if (n4 == 0) return MUIR_OK;
  int64_t blocks = (n4 + 255) / 256;
  if (blocks > 148 * 32) blocks = 148 * 32;
  Launch L_("state_init", static_cast<cudaStream_t>(stream));
  muir::state_init_kernel<<<(unsigned)blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<float4*>(S), reinterpret_cast<const float4*>(S_src), n4);
  return cuda_check("state_init launch");
}

int muir_row_scale(const float* S, int64_t n_seq, int32_t H, int32_t dk, int32_t dv, float exponent, float eps, float* r,
                   void* stream) {
  g_err.clear();
  if (!S || !r) return fail(MUIR_ERR_INVALID_ARG, "row_scale: S or r is NULL");
  if (n_seq <= 0 || H <= 0 || !dim_ok(dk) || !dim_ok(dv))
    return fail(MUIR_ERR_UNSUPPORTED, "row_scale: unsupported sizes n_seq=%lld H=%d dk=%d dv=%d", (long long)n_seq, H,
                dk, dv);
  if (!(exponent >= 0.f) || !(eps >= 0.f)) return fail(MUIR_ERR_INVALID_ARG, "row_scale: exponent and eps must be >= 0");
  Launch L_("row_scale", static_cast<cudaStream_t>(stream));
  muir::row_scale_kernel<<<(unsigned)(H * dk), 256, 0, static_cast<cudaStream_t>(stream)>>>(S, n_seq, H, dk, dv,
                                                                                            exponent, eps, r);
  return cuda_check("row_scale launch");
}

int muir_apply_map(const float* Phi, const float* Psi, const float* S_in, float* S_out, int64_t n_seq, int32_t H,
                   int32_t dk, int32_t dv, void* stream) {
  g_err.clear();
  if (!Phi || !Psi || !S_out) return fail(MUIR_ERR_INVALID_ARG, "apply_map: Phi, Psi or S_out is NULL");
  if (n_seq < 0 || H <= 0 || !dim_ok(dk) || !dim_ok(dv))
    return fail(MUIR_ERR_UNSUPPORTED, "apply_map: unsupported sizes n_seq=%lld H=%d dk=%d dv=%d", (long long)n_seq, H,
                dk, dv);
  if (S_in && S_in == S_out) return fail(MUIR_ERR_INVALID_ARG, "apply_map: S_in and S_out must differ");
  const int64_t total = n_seq * H * (int64_t)dk * dv;
  if (total == 0) return MUIR_OK;
  int64_t blocks = (total + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  Launch L_("apply_map", static_cast<cudaStream_t>(stream));
  muir::apply_map_kernel<<<(unsigned)blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(Phi, Psi, S_in, S_out,
                                                                                         n_seq * H, dk, dv);
  return cuda_check("apply_map launch");
}

int muir_decode_step(const muir_decode_args* a, void* stream) {
  g_err.clear();
  if (!a) return fail(MUIR_ERR_INVALID_ARG, "decode: args is NULL");
  if (a->n_seq == 0) return MUIR_OK;  // nothing to do (empty tensors may carry NULL pointers)
  if (!a->S || !a->q || !a->k || !a->v || !a->e || !a->w || !a->log_alpha || !a->r || !a->y)
    return fail(MUIR_ERR_INVALID_ARG, "decode: a required pointer is NULL");
  if (a->n_seq < 0 || a->H <= 0 || !dim_ok(a->dk) || !dim_ok(a->dv))
    return fail(MUIR_ERR_UNSUPPORTED, "decode: unsupported sizes H=%d dk=%d dv=%d", a->H, a->dk, a->dv);
  if (a->dtype != MUIR_F32 && a->dtype != MUIR_BF16) return fail(MUIR_ERR_UNSUPPORTED, "decode: dtype %d", a->dtype);
  if (a->r_seq_stride < 0) return fail(MUIR_ERR_INVALID_ARG, "decode: negative r_seq_stride");
  const void* ptrs[] = {a->S, a->q, a->k, a->v, a->e, a->w, a->g, a->z, a->log_alpha, a->r, a->y};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(MUIR_ERR_INVALID_ARG, "decode: pointer not 16-byte aligned");
  if (a->n_seq == 0) return MUIR_OK;
  muir::DecodeParams p{a->n_seq, a->H, a->dk, a->dv, a->S, a->q, a->k, a->v, a->e, a->w, a->g, a->z,
                       a->log_alpha, a->r, a->r_seq_stride, a->y};
  const int64_t blocks = a->n_seq * a->H * (a->dv / 32);
  if (blocks > 0x7fffffff) return fail(MUIR_ERR_UNSUPPORTED, "decode: too many rows");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool bf = a->dtype == MUIR_BF16;
  Launch L_("decode_step", s);
#define MUIR_DECODE(DK)                                                                  \
  if (bf)                                                                                \
    muir::decode_step_kernel<DK, __nv_bfloat16><<<(unsigned)blocks, 128, 0, s>>>(p);     \
  else                                                                                   \
    muir::decode_step_kernel<DK, float><<<(unsigned)blocks, 128, 0, s>>>(p);
  switch (a->dk) {
    case 32: MUIR_DECODE(32) break;
    case 64: MUIR_DECODE(64) break;
    default: MUIR_DECODE(128) break;
  }
#undef MUIR_DECODE
  return cuda_check("decode launch");
}

// Diagnostic entry point: D[128,N] = A[128,K] * B[K,N] through the tensor-core
// operand layouts the chunk kernels use. a_mn/b_mn select MN-major staging,
// nsplit is 1 or 3. Not part of the operator.
int muir_selftest_gemm(const float* A, const float* B, float* D, int32_t N, int32_t K, int32_t a_mn, int32_t b_mn,
                       int32_t nsplit, void* stream) {
  g_err.clear();
  if (!A || !B || !D) return fail(MUIR_ERR_INVALID_ARG, "selftest: NULL pointer");
  if (N < 16 || N > 256 || N % 16 || K < 16 || K > 128 || K % 16 || (nsplit != 1 && nsplit != 3))
    return fail(MUIR_ERR_UNSUPPORTED, "selftest: N=%d K=%d nsplit=%d", N, K, nsplit);
  const size_t smem = 2u * (128u * K * 2u) + 2u * ((size_t)N * K * 2u);
  if (cudaFuncSetAttribute(muir::selftest_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return cuda_check("selftest attribute");
  Launch L_("selftest_gemm", static_cast<cudaStream_t>(stream));
  muir::selftest_gemm_kernel<<<1, 128, smem, static_cast<cudaStream_t>(stream)>>>(A, B, D, N, K, a_mn, b_mn, nsplit);
  return cuda_check("selftest launch");
}

// Diagnostic entry point: one bounded wait on an mbarrier that completes
// (arrive != 0) or that nothing ever completes (arrive == 0), given up after
// limit_ns. out (device int) receives 1 if the wait saw the phase complete.
int muir_selftest_wait(uint64_t limit_ns, int32_t arrive, int32_t* out, void* stream) {
  g_err.clear();
  if (!out) return fail(MUIR_ERR_INVALID_ARG, "selftest_wait: out is NULL");
  if (limit_ns > muir::kWaitLimitNs)
    return fail(MUIR_ERR_INVALID_ARG, "selftest_wait: limit %llu ns above the library's %llu ns",
                (unsigned long long)limit_ns, (unsigned long long)muir::kWaitLimitNs);
  Launch L_("selftest_wait", static_cast<cudaStream_t>(stream));
  muir::selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns, arrive, out);
  return cuda_check("selftest_wait launch");
}

// Diagnostic entry point: D[128,N] = A[128,K] B[K,N] (bf16 A and B row-major,
// fp32 D) through 128-byte-swizzled operand tiles, loaded by TMA (mode 1) or by
// the threads (mode 0; mode 2 with A stored as the MN-major operand). K in
// {64, 128}, N in {64, 128, 256}.
int muir_selftest_sw128(const void* A, const void* B, float* D, int32_t N, int32_t K, int32_t mode, void* stream) {
  g_err.clear();
  if (!A || !B || !D) return fail(MUIR_ERR_INVALID_ARG, "selftest_sw128: NULL pointer");
  if ((K != 64 && K != 128) || (N != 64 && N != 128 && N != 256))
    return fail(MUIR_ERR_UNSUPPORTED, "selftest_sw128: N=%d K=%d", N, K);
  if (!aligned16(A) || !aligned16(B)) return fail(MUIR_ERR_INVALID_ARG, "selftest_sw128: misaligned pointer");
  if (mode < 0 || mode > 2) return fail(MUIR_ERR_INVALID_ARG, "selftest_sw128: mode %d", mode);
  const bool use_tma = mode == 1;
  CUtensorMap ta{}, tb{};
  if (use_tma && (!muir_host::make_tmap_bf16(&ta, A, 128, K, K, 128) ||
                  !muir_host::make_tmap_bf16(&tb, B, K, N, N, (uint32_t)K)))
    return fail(MUIR_ERR_CUDA, "selftest_sw128: tensor map encoding failed");
  const size_t smem = 1024u + (size_t)(K / 64) * 16384u + (size_t)(N / 64) * K * 128u;
  if (cudaFuncSetAttribute(muir::selftest_sw128_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return cuda_check("selftest_sw128 attribute");
  Launch L_("selftest_sw128", static_cast<cudaStream_t>(stream));
  muir::selftest_sw128_kernel<<<1, 128, smem, static_cast<cudaStream_t>(stream)>>>(
      ta, tb, static_cast<const __nv_bfloat16*>(A), static_cast<const __nv_bfloat16*>(B), D, N, K, mode);
  return cuda_check("selftest_sw128 launch");
}

void muir_profile_begin(void) {
  for (auto& r : g_prof.recs) {
    g_prof.pool.push_back(r.a);
    g_prof.pool.push_back(r.b);
  }
  g_prof.recs.clear();
  g_prof.on = true;
}

int muir_profile_end(char* names_buf, size_t names_cap, float* ms, int64_t* launches, int max_entries) {
  g_prof.on = false;
  std::vector<std::string> names;
  std::vector<double> tot;
  std::vector<int64_t> cnt;
  for (auto& r : g_prof.recs) {
    if (cudaEventSynchronize(r.b) != cudaSuccess) return -1;
    float t = 0.f;
    if (cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess) return -1;
    const std::string key = (r.phase[0] ? std::string(r.phase) + ":" : std::string()) + r.name;
    size_t k = 0;
    while (k < names.size() && names[k] != key) ++k;
    if (k == names.size()) {
      names.emplace_back(key);
      tot.push_back(0.0);
      cnt.push_back(0);
    }
    tot[k] += t;
    cnt[k] += 1;
  }
  std::string joined;
  const int n = (int)names.size() < max_entries ? (int)names.size() : max_entries;
  for (int i = 0; i < n; ++i) {
    joined += names[i];
    joined += '\n';
    ms[i] = (float)tot[i];
    launches[i] = cnt[i];
  }
  if (names_buf && names_cap) {
    const size_t m = joined.size() < names_cap - 1 ? joined.size() : names_cap - 1;
    memcpy(names_buf, joined.data(), m);
    names_buf[m] = 0;
  }
  return n;
}

int64_t muir_launch_count(void) { return g_prof.launches; }

}  // extern "C"

#include "api_chunk.inc"
#include "api_gate.inc"

// ---------------------------------------------------------------------------
// Allocation-free chunkwise forward.
//
// Some callers cannot allocate device memory: a host that embeds this library
// as a plug-in and hands it only its input and output buffers, or a
// latency-critical loop that must not call cudaMalloc/cudaFree because those
// calls can synchronise the whole device. For them the forward pass can run on
// a scratch area compiled into the library: a file-scope device array of
// kNoAllocScratchBytes, which every GPU that loads the library holds until the
// process exits.
// ---------------------------------------------------------------------------
namespace {
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB
}

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
std::mutex g_noalloc_mu;
constexpr int kMaxDevices = 64;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device. In host code the
// array's name is only a host-side stand-in, so the address must come from
// cudaGetSymbolAddress, once per device, with that device current.
int noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cuda_check("chunk_fwd_noalloc: cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(MUIR_ERR_UNSUPPORTED, "chunk_fwd_noalloc: device ordinal %d", dev);
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess)
      return fail(MUIR_ERR_CUDA, "chunk_fwd_noalloc: cudaGetSymbolAddress: %s", cudaGetErrorString(e));
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return MUIR_OK;
}
}  // namespace

extern "C" int muir_chunk_fwd_noalloc(const muir_chunk_args* a, void* y, float* S_T, void* stream) {
  g_err.clear();
  int rc = validate_chunk_args(a, "chunk_fwd_noalloc");
  if (rc) return rc;
  if (a->flags != 0) return fail(MUIR_ERR_INVALID_ARG, "chunk_fwd_noalloc: flags must be 0");
  const size_t need = muir_chunk_fwd_workspace(a);
  if (need > kNoAllocScratchBytes)
    return fail(MUIR_ERR_UNSUPPORTED,
                "chunk_fwd_noalloc: this problem needs %zu bytes of scratch but the built-in scratch holds %zu; "
                "use muir_chunk_fwd with a caller-provided workspace",
                need, kNoAllocScratchBytes);
  void* ws = nullptr;
  if ((rc = noalloc_scratch(&ws))) return rc;
  return muir_chunk_fwd(a, y, S_T, ws, kNoAllocScratchBytes, stream);
}
