/*
 * muir_profile.h — diagnostics of libmuir.so (not part of the operator API).
 *
 * Kernel timing: between muir_profile_begin() and muir_profile_end(), every
 * kernel the library launches is bracketed by a pair of CUDA events recorded on
 * the stream it is launched on. muir_profile_end() synchronises those events and
 * returns, per kernel name, the number of launches and the summed device time.
 * Profiling is process-wide and not thread-safe; it costs two event records per
 * launch, so time throughput with it off.
 *
 * muir_launch_count(): number of kernels the library has launched since load.
 *
 * muir_selftest_gemm(): D[128,N] = A[128,K] * B[K,N] (fp32 row-major device
 * buffers) through the tensor-core operand layouts the chunk kernels use;
 * a_mode/b_mode bit 0 = MN-major operand, bit 1 = read through the transposed
 * view of a tile written in the other arrangement; nsplit 1 or 3 bf16 passes.
 *
 * muir_selftest_wait(): the give-up path of the library's bounded device
 * waits. One warp waits for phase 0 of an mbarrier in its own shared memory,
 * through the same wait routine the kernels use but with a limit of limit_ns
 * (at most the library's one second). With arrive != 0 the phase completes
 * before the wait; with arrive == 0 nothing ever completes it, so the wait runs
 * out, sets the status word that muir_device_status() reports as
 * MUIR_ERR_TIMEOUT, and the kernel returns. No copy or tensor-core operation is
 * in flight, so the give-up leaves nothing behind. *out (a device int32)
 * receives 1 if the wait saw the phase complete, else 0.
 *
 * muir_selftest_sw128(): D[128,N] = A[128,K] * B[K,N] with bf16 A and B
 * (row-major device buffers) and fp32 D, through 128-byte-swizzled operand
 * tiles: A as the K-major operand and B as the MN-major one, loaded by TMA boxes
 * (mode 1) or written by the threads in the same layout (mode 0); mode 2 has the
 * threads store A transposed, as the MN-major operand (rows = K). K in {64, 128},
 * N in {64, 128, 256}; another mode is MUIR_ERR_INVALID_ARG.
 */
#ifndef MUIR_PROFILE_H
#define MUIR_PROFILE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

void muir_profile_begin(void);
/* names: '\n'-separated kernel names written into names_buf (NUL-terminated);
 * ms[i], launches[i]: totals for the i-th name. Returns the number of names
 * (at most max_entries), or -1 on a CUDA error. */
int muir_profile_end(char* names_buf, size_t names_cap, float* ms, int64_t* launches, int max_entries);
int64_t muir_launch_count(void);
int muir_selftest_gemm(const float* A, const float* B, float* D, int32_t N, int32_t K, int32_t a_mode,
                       int32_t b_mode, int32_t nsplit, void* stream);
int muir_selftest_wait(uint64_t limit_ns, int32_t arrive, int32_t* out, void* stream);
int muir_selftest_sw128(const void* A, const void* B, float* D, int32_t N, int32_t K, int32_t mode, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MUIR_PROFILE_H */
