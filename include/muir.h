/*
 * muir.h — C ABI of the Muir gated delta-rule operator library (libmuir.so),
 * hand-written CUDA for NVIDIA B200 (sm_100a).
 *
 * The operator (arXiv 2611.08376, "Muir: Linear Attention with
 * Sensitivity-Allocated Gating and Matched-Filter Readout", abstract "Full
 * text"; openai-hub article, sections on the matched-filter readout and on
 * the TPU chunkwise algorithm). Per batch b, head h, token t:
 *
 *   x_t = Diag(alpha_t) S_{t-1}                     channel-wise decay of the rows of S
 *   p_t = x_t^T k_t                                 prediction for the incoming key
 *   S_t = x_t - (e_t*k_t) p_t^T + k_t (w_t*v_t)^T   gated erase of the prediction, gated write
 *   o_t = S_t^T (r * g_t * q_t)                     matched-filter readout: static row scale r,
 *                                                   dynamic per-token query gate g_t
 *   y_t = z_t * o_t                                 output gate (z may be omitted: y = o)
 *
 * S is a dk x dv fp32 matrix per (sequence, head). alpha is passed as
 * log_alpha <= 0 (fp32). q and k are expected to be already activated and
 * unit-normalised by the caller; the operator does not normalise.
 *
 * Conventions for every entry point:
 *   - Pointers are CUDA device pointers owned by the caller; the library never
 *     allocates, frees or retains them. Scratch memory ("workspace") is passed
 *     in by the caller after a size query.
 *   - Tensors are dense, row-major, in the layouts stated per argument, and
 *     every pointer must be 16-byte aligned.
 *   - "dtype" selects the element type of q, k, v, e, w, g, z, y and of the
 *     gradients of those: MUIR_F32 (float) or MUIR_BF16 (bfloat16). log_alpha,
 *     r, states and their gradients are always float.
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t, NULL = the
 *     legacy default stream). Return values report argument validation and
 *     launch errors only; a kernel's bounded waits that ran out are reported by
 *     muir_device_status().
 *   - Return: MUIR_OK (0) or one of the MUIR_ERR_* codes below; a message for
 *     the calling thread is available from muir_last_error(). Nothing is thrown
 *     across this interface.
 *   - Supported sizes: dk, dv in {32, 64, 128}; chunk in {64, 128, 256};
 *     T % chunk == 0 (callers pad with identity tokens: log_alpha = 0, k = 0,
 *     e = 0, w = 0, which leave the state unchanged).
 */
#ifndef MUIR_H
#define MUIR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MUIR_OK 0
#define MUIR_ERR_INVALID_ARG 1 /* null pointer, bad stride/alignment, inconsistent sizes */
#define MUIR_ERR_UNSUPPORTED 2 /* valid but unsupported size, chunk or dtype */
#define MUIR_ERR_WORKSPACE 3   /* workspace pointer NULL/misaligned or smaller than the query */
#define MUIR_ERR_CUDA 4        /* a CUDA runtime call failed (launch, attribute) */
#define MUIR_ERR_TIMEOUT 5     /* a bounded device wait expired (from muir_device_status) */
#define MUIR_ERR_BOUNDS 6      /* checking builds (-DMUIR_CHECK) only: a device index failed its bounds
                                  check; the access was skipped (from muir_device_status) */

#define MUIR_F32 0
#define MUIR_BF16 1

/* Bits of muir_chunk_args.flags (every other bit must be 0). */
#define MUIR_SAVE_FOR_BWD 1 /* muir_chunk_fwd: also leave in the workspace what muir_chunk_bwd needs */
#define MUIR_USE_SAVED 2    /* muir_chunk_bwd: the workspace holds it; skip the recomputation */

/* Inputs of the chunkwise forward and backward passes. */
typedef struct muir_chunk_args {
  int64_t B;      /* batch size (independent sequences) */
  int64_t T;      /* tokens per sequence; T % chunk == 0 */
  int32_t H;      /* heads */
  int32_t dk;     /* key dimension = rows of the state */
  int32_t dv;     /* value dimension = columns of the state */
  int32_t chunk;  /* chunk length C of the chunkwise algorithm: 64, 128 or 256 */
  int32_t dtype;  /* MUIR_F32 or MUIR_BF16 */
  int32_t flags;  /* 0, or MUIR_SAVE_FOR_BWD (forward) / MUIR_USE_SAVED (backward) */
  const void* q;  /* [B,T,H,dk] query (activated, unit-norm) */
  const void* k;  /* [B,T,H,dk] key (activated, unit-norm) */
  const void* v;  /* [B,T,H,dv] value */
  const void* e;  /* [B,T,H,dk] erase gate, acts on key rows */
  const void* w;  /* [B,T,H,dv] write gate, acts on value columns */
  const void* g;  /* [B,T,H,dk] dynamic query (read) gate, or NULL for the static-only
                     readout (g = 1: the query is scaled by r alone; openai-hub article,
                     matched-filter section, compares static and dynamic readouts) */
  const void* z;  /* [B,T,H,dv] output gate, or NULL for none */
  const float* log_alpha; /* [B,T,H,dk] log of the channel decay, <= 0 */
  const float* r; /* [H,dk] static matched-filter row scale */
  const float* S0;/* [B,H,dk,dv] initial state, or NULL for zeros */
} muir_chunk_args;

/*
 * Chunkwise-parallel forward pass (openai-hub article, section on the TPU
 * chunkwise algorithm; liuch.name post, bullet "Numerically-stable,
 * large-chunk parallel kernel"): intra-chunk decay products are
 * boundary-pivoted and multiplicative (each factor in [0,1], no division), the
 * unit-lower-triangular chunk system is inverted by a recursive block method on
 * the tensor cores, and the state is passed from chunk to chunk on chip.
 *   y   [B,T,H,dv] output (dtype).
 *   S_T [B,H,dk,dv] final state, or NULL if not wanted.
 *   ws  workspace of at least muir_chunk_fwd_workspace(a) bytes, 256-byte
 *       aligned; contents on entry are ignored.
 */
/*
 * muir_chunk_fwd_workspace: bytes of device scratch that muir_chunk_fwd needs
 * for these arguments (openai-hub article, section "为 TPU 重写长序列并行算法":
 * the chunkwise algorithm keeps per-chunk intermediates, which the pages' XLA
 * version wrote to HBM; here they are the per-unit decay products, Gram and T
 * images, chunk maps and chunk-start states). Only the sizes, chunk, dtype and
 * flags of *a are read; with MUIR_SAVE_FOR_BWD it returns the size that also
 * holds what the backward pass reuses. Returns 0 when the arguments are
 * invalid (muir_last_error() says why) and for empty problems (B = 0 or T = 0),
 * which need no workspace. The caller allocates and owns the workspace.
 */
size_t muir_chunk_fwd_workspace(const muir_chunk_args* a);
int muir_chunk_fwd(const muir_chunk_args* a, void* y, float* S_T, void* ws, size_t ws_bytes,
                   void* stream);
/*
 * Saving for the backward pass (a packaging choice of the library; the pages
 * describe the backward only as a parallel update). With MUIR_SAVE_FOR_BWD in
 * a->flags, muir_chunk_fwd needs a workspace of muir_chunk_fwd_workspace(a)
 * bytes, which then equals muir_chunk_bwd_workspace(a), and leaves in it the
 * per-unit decay products, Gram and T images, chunk maps, W, Ut and the
 * unit-start states. It works on units of min(chunk, 128) tokens (the
 * backward's units; for chunk 256 the state is carried every 128 tokens, which
 * is the same map). A following muir_chunk_bwd with MUIR_USE_SAVED in its
 * flags (otherwise the same arguments, the same inputs and the same workspace,
 * untouched in between) then skips the forward recomputation. Memory: about
 * 1.1 MB per 128 tokens per (batch, head) at dk = dv = 128.
 */

/* Gradients for muir_chunk_bwd. Outputs are written (not accumulated). */
typedef struct muir_chunk_grads {
  const void* dy;      /* [B,T,H,dv] cotangent of y (dtype) */
  const float* dS_T;   /* [B,H,dk,dv] cotangent of the final state, or NULL for zeros */
  void* dq;            /* [B,T,H,dk] (dtype) */
  void* dk;            /* [B,T,H,dk] (dtype) */
  void* dv;            /* [B,T,H,dv] (dtype) */
  void* de;            /* [B,T,H,dk] (dtype) */
  void* dw;            /* [B,T,H,dv] (dtype) */
  void* dg;            /* [B,T,H,dk] (dtype); may be NULL (and is ignored) when g is NULL */
  void* dz;            /* [B,T,H,dv] (dtype), or NULL; ignored when z is NULL */
  float* dlog_alpha;   /* [B,T,H,dk]; d/d(alpha) = dlog_alpha / alpha */
  float* dS0;          /* [B,H,dk,dv], or NULL */
  float* dr;           /* [H,dk], or NULL */
} muir_chunk_grads;

/*
 * Backward pass of muir_chunk_fwd with the same arguments. The per-chunk
 * states are recomputed (a forward sweep into the workspace), then one reverse
 * sweep carries the state cotangent, and chunk-parallel kernels form every
 * input gradient (arXiv abstract: a parallel update for training).
 *   ws  workspace of at least muir_chunk_bwd_workspace(a) bytes; with
 *       MUIR_USE_SAVED in a->flags, the workspace a forward pass with
 *       MUIR_SAVE_FOR_BWD filled (see above).
 */
/*
 * muir_chunk_bwd_workspace: bytes of device scratch muir_chunk_bwd needs (the
 * same section of the openai-hub article: the backward pass recomputes the
 * per-chunk states and keeps the cotangents of the chunk quantities between
 * its kernels). Only the sizes, chunk and dtype of *a are read. Returns 0 when
 * the arguments are invalid and for empty problems. The caller allocates and
 * owns the workspace; it equals muir_chunk_fwd_workspace() of the same
 * arguments with MUIR_SAVE_FOR_BWD.
 */
size_t muir_chunk_bwd_workspace(const muir_chunk_args* a);
int muir_chunk_bwd(const muir_chunk_args* a, const muir_chunk_grads* gr, void* ws, size_t ws_bytes,
                   void* stream);

/*
 * Allocation-free variant of muir_chunk_fwd (the pages have no counterpart;
 * this is a packaging choice of the library). For callers that cannot allocate
 * device memory — a host that embeds the library as a plug-in and owns all
 * allocations, or a latency-critical loop that must not call cudaMalloc or
 * cudaFree because they can synchronise the device — the forward pass runs on
 * a 32 MiB scratch area compiled into the library (every GPU that loads the
 * library holds it until the process exits). The caller still passes inputs
 * and outputs exactly as for muir_chunk_fwd; this call allocates nothing.
 *   - a->flags must be 0 (MUIR_ERR_INVALID_ARG otherwise): nothing can be saved
 *     for a backward pass in the library's scratch.
 *   - Problems whose muir_chunk_fwd_workspace() exceeds 32 MiB are rejected
 *     with MUIR_ERR_UNSUPPORTED before any GPU work.
 *   - The first call on a device looks up the scratch address with
 *     cudaGetSymbolAddress (once per device, with that device current); make
 *     that first call before any stream capture on the device.
 *   - The scratch address is cached per device for the life of the process:
 *     do not keep using the library on a device after cudaDeviceReset (or any
 *     other teardown of its primary context), which may move the area.
 *   - All calls on a device share the one scratch area and it keeps the last
 *     call's contents; the kernels write every scratch byte they read within
 *     the same call, so nothing needs clearing. Calls that overlap on the GPU
 *     (e.g. on two streams at once) race on the scratch: serialise them.
 */
int muir_chunk_fwd_noalloc(const muir_chunk_args* a, void* y, float* S_T, void* stream);

/*
 * Sequence segments (a scan split along T; the pages have no counterpart). The
 * chunkwise forward is an affine map of its start state, S_T = Phi S0 + Psi.
 * muir_chunk_segment_map returns that map for a whole segment (the chunk maps
 * of its units of min(chunk, 128) tokens, composed in order on the tensor
 * cores): Phi [B,H,dk,dk] and Psi [B,H,dk,dv] fp32 (device, caller-owned), so
 * that ranks holding consecutive segments can exchange maps, and each one
 * start from its predecessors' maps applied to the initial state. a->S0 is
 * ignored; a->flags must be 0. Workspace: muir_chunk_segment_map_workspace(a).
 * muir_apply_map computes S_out = Phi S_in + Psi (S_in NULL: S_out = Psi) in
 * fp32 on [n_seq,H] maps; S_in and S_out must not alias.
 */
size_t muir_chunk_segment_map_workspace(const muir_chunk_args* a);
int muir_chunk_segment_map(const muir_chunk_args* a, float* Phi, float* Psi, void* ws, size_t ws_bytes, void* stream);
int muir_apply_map(const float* Phi, const float* Psi, const float* S_in, float* S_out, int64_t n_seq, int32_t H,
                   int32_t dk, int32_t dv, void* stream);

/* One recurrent step for n_seq independent sequences (streaming decode,
 * openai-hub article, section on 10M-token streaming). */
typedef struct muir_decode_args {
  int64_t n_seq;       /* number of (sequence, layer) rows */
  int32_t H, dk, dv;
  int32_t dtype;       /* of q,k,v,e,w,g,z,y */
  float* S;            /* [n_seq,H,dk,dv] state, updated in place */
  const void* q;       /* [n_seq,H,dk] */
  const void* k;       /* [n_seq,H,dk] */
  const void* v;       /* [n_seq,H,dv] */
  const void* e;       /* [n_seq,H,dk] */
  const void* w;       /* [n_seq,H,dv] */
  const void* g;       /* [n_seq,H,dk], or NULL for the static-only readout (g = 1) */
  const void* z;       /* [n_seq,H,dv] or NULL */
  const float* log_alpha; /* [n_seq,H,dk] */
  const float* r;      /* [H,dk] when r_seq_stride == 0, else row n at r + n*r_seq_stride */
  int64_t r_seq_stride;/* elements between consecutive rows' r (0 = shared, H*dk = per row) */
  void* y;             /* [n_seq,H,dv] output */
} muir_decode_args;

/* Reads and writes each state element exactly once (memory-bound). */
int muir_decode_step(const muir_decode_args* a, void* stream);

/* Set up the recurrent state (openai-hub article, section "1000 万 Token，KV
 * Cache 已经装不下了": the model carries a fixed-size fp32 state per head, about
 * 25 MB over 24 layers of 16 heads of 128 x 128, in place of a KV cache):
 * S [n_seq,H,dk,dv] fp32 := S_src, or zeros when S_src is NULL. Both are device
 * pointers owned by the caller, 16-byte aligned; S == S_src is allowed (a no-op
 * copy), other overlaps are not. dk, dv in {32, 64, 128}. n_seq = 0 launches
 * nothing. Returns MUIR_ERR_INVALID_ARG for a NULL S or a misaligned pointer,
 * MUIR_ERR_UNSUPPORTED for n_seq < 0, H <= 0 or dk, dv outside {32, 64, 128},
 * and MUIR_ERR_CUDA if the launch fails. */
int muir_state_init(float* S, const float* S_src, int64_t n_seq, int32_t H, int32_t dk, int32_t dv,
                    void* stream);

/* Static matched-filter row scale from measured row energies (openai-hub
 * article, matched-filter section: the static readout weights each state row
 * by an inverse fractional power of its expected energy; 0.5 is the inverse
 * square root). For states S [n_seq,H,dk,dv] fp32 (device), e.g. collected
 * along a calibration stream, with E[h,i] = mean over (n, j) of S[n,h,i,j]^2:
 *     r[h,i] = (E[h,i] + eps)^(-exponent)          r [H,dk] fp32 (device)
 * The sums are accumulated in fp64. exponent, eps >= 0. The scale is returned
 * as is (no normalisation), for the caller to rescale if wanted. */
int muir_row_scale(const float* S, int64_t n_seq, int32_t H, int32_t dk, int32_t dv, float exponent, float eps, float* r,
                   void* stream);

/* Fused low-rank gate projection (openai-hub article, section "五套门控被压进一个
 * 低秩投影" and its table; liuch.name post, second bullet): the five gate
 * tensors of the operator from the layer input x with one shared down-projection
 * of total rank 512, sliced 64 / 64 / 128 / 128 / 128 for the decay, erase,
 * output, write and dynamic-read gates, each slice with its own up-projection:
 *     h = x W_down,   u_j = h[:, slice_j] U_j
 *     log_alpha = log sigmoid(u_decay)   e = sigmoid(u_erase)   z = sigmoid(u_out)
 *     w = sigmoid(u_write)               g = sigmoid(u_read)
 * Arguments (device pointers, row-major, every pointer 16-byte aligned; the
 * element type of every array but log_alpha is `dtype`, log_alpha is float):
 *     x        [n_tokens][d_model]          w_down  [d_model][512]
 *     u_decay, u_erase [64][ok]             u_out, u_write [128][ov]
 *     u_read   [128][ok]
 *     log_alpha, e, g  [n_tokens][ok]  (out)   z, w  [n_tokens][ov]  (out)
 * ok = H*d_k and ov = H*d_v, so the outputs are in the operator's [B,T,H,d]
 * layout with the tokens flattened. d_model must be a multiple of 64, ok and ov
 * multiples of 256 (else MUIR_ERR_UNSUPPORTED). n_tokens may be 0 (no launch;
 * the pointers are not read and may be NULL) or any size (a ragged last tile is
 * masked). Otherwise a NULL or misaligned pointer gives MUIR_ERR_INVALID_ARG. h is accumulated in fp32 and kept
 * at fp32 accuracy into the up-projections; the activations are evaluated in
 * fp32. Enqueued on `stream`; the caller owns every buffer. */
int muir_gate_proj(const void* x, const void* w_down, const void* u_decay, const void* u_erase, const void* u_out,
                   const void* u_write, const void* u_read, float* log_alpha, void* e, void* z, void* w, void* g,
                   int64_t n_tokens, int32_t d_model, int32_t ok, int32_t ov, int32_t dtype, void* stream);

/* Synchronises `stream`, then returns and clears the device-side status word:
 * MUIR_OK, or MUIR_ERR_TIMEOUT if a kernel's bounded wait expired since the
 * last call (that kernel's outputs are then invalid), MUIR_ERR_BOUNDS (checking
 * builds only) if an index failed its bounds check, or MUIR_ERR_CUDA. */
int muir_device_status(void* stream);

/* Message describing the last error on the calling thread ("" if none). */
const char* muir_last_error(void);

/* Library ABI version (major*100 + minor). */
int muir_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MUIR_H */
