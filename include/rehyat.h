/*
 * rehyat.h -- C ABI of the B200 (sm_100a) implementation of ReHyAt's
 * temporally chunked hybrid attention forward.
 *
 * Source of every operation: "ReHyAt: Recurrent Hybrid Attention for Video
 * Diffusion Transformers" (Ghafoorian & Habibian, arXiv 2601.04342):
 *   §3.1  linear attention y_i = phi(q_i) sum_j phi(k_j) v_j^T / phi(q_i) sum_j phi(k_j),
 *         the two sums cached independently of i; phi non-negative, 1 + elu.
 *   §3.2  hybrid output y = (a^S + a^L) / (n^S + n^L) (joint normaliser);
 *         chunk sets T^S_t, T^L_t with and without overlap;
 *         polynomial feature map phi(x) = [psi_1(x)^1, ..., psi_P(x)^P].
 *   §3.3  Recurrent HyAt: T^L_t = { j < max(tN' - T_o HW, 0) },
 *         T^S_t = { max(tN' - T_o HW, 0) <= j < (t+1)N' }.
 *
 * Readings taken where the text is silent (the paper's prose around the
 * equations is lost):
 *   - N' = chunk_frames * S_tok; chunk t owns queries [tN', min((t+1)N', N)).
 *   - tokens are frame-major: j = f * S_tok + spatial index; N = F * S_tok.
 *   - the last chunk is ragged when F is not a multiple of chunk_frames.
 *   - phi(x) = [psi(x), psi(x)^2] with psi = 1 + elu on both q and k (P = 2,
 *     D' = 2d): the only concrete psi the paper gives.  The learned maps of
 *     §4.3 / §7.1 (two-layer MLP, separate phi_q and phi_k) are the
 *     rehyat_phi_mlp / _phi / _mlp entry points below.
 *   - softmax weight exp(q.k / sqrt(d)).
 *   - every call computes the §3.3 (causal / recurrent) sets, so the parallel
 *     form and the step form compute the same function; rehyat_forward_ex
 *     also offers the §3.2 bidirectional sets.
 *
 * Conventions for every entry point:
 *   - Tensors are dense, row-major, in DEVICE memory owned by the caller
 *     (rehyat_forward_host alone takes host q, k, v, out): q, k, v, out are
 *     [B, H, N, d] (d fastest), or [B, N, H, d] where a `layout` argument
 *     says so.  bf16 entry points take `const void*` pointing at IEEE
 *     bfloat16 data; _f32 ones take float.  All device pointers must be
 *     16-byte aligned (TMA requirement).
 *   - d must be 64 or 128 (REHYAT_EUNSUPPORTED otherwise).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Calls are asynchronous: they validate, launch and return;
 *     outputs are valid once the stream reaches that point.  No host sync.
 *   - Validation failures return a status and launch nothing.  Launch
 *     failures return REHYAT_ECUDA.  Entry points without a `workspace`
 *     argument allocate stream-ordered scratch (cudaMallocAsync /
 *     cudaFreeAsync on `stream`); the _ws variants allocate nothing.
 *   - Device-side waits are bounded (about 2 s).  A wait that runs out sets
 *     a device error word, the kernel returns early (its outputs are then
 *     invalid), and rehyat_device_status() reports REHYAT_ETIMEOUT.
 *   - Results are deterministic: no atomics on the data path.
 *   - Multiple calls may run concurrently on different streams.
 *   - CUDA graphs: the entry points that take a caller workspace allocate
 *     nothing and never synchronise the host, so their launches can be
 *     captured into a CUDA graph.  Make one eager call per kernel variant
 *     and device first (it sets the kernel's shared-memory limit once).
 */
#ifndef REHYAT_H
#define REHYAT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  REHYAT_OK = 0,
  REHYAT_EINVAL = 1,        /* bad argument: null/misaligned pointer, size < 1, overflow */
  REHYAT_EUNSUPPORTED = 2,  /* valid but not implemented here (d not in {64,128}) */
  REHYAT_ENOMEM = 3,        /* workspace allocation failed / workspace too small */
  REHYAT_ECUDA = 4,         /* a CUDA runtime/driver call or launch failed */
  REHYAT_ETIMEOUT = 5       /* a bounded device-side wait ran out (see rehyat_device_status) */
} rehyat_status;

/* Human-readable name of a status code (static string, never NULL). */
const char* rehyat_status_string(int status);

/* ---------------------------------------------------------------------- *
 * Parallel form (§3.2 joint normaliser over the §3.3 sets), whole video.  *
 * ---------------------------------------------------------------------- */

/* bf16 forward on tensor cores (tcgen05/TMEM, TMA).
 * q, k, v: [B,H,N,d] bf16 with N = F*S_tok.  out: [B,H,N,d] bf16.
 * chunk_frames = T_c >= 1, overlap_frames = T_o >= 0 (any value, also >= T_c).
 * Arithmetic: bf16 operands, fp32 accumulation, fp32 softmax and combine;
 * the linear state is kept in fp32 and fed to the tensor cores as a bf16
 * hi + lo pair. */
int rehyat_forward(const void* q, const void* k, const void* v,
                   int B, int H, int F, int S_tok, int d,
                   int chunk_frames, int overlap_frames,
                   void* out, void* stream);

/* Bytes of scratch rehyat_forward_ws needs for this shape. */
int rehyat_forward_workspace_bytes(int B, int H, int F, int S_tok, int d,
                                   int chunk_frames, int overlap_frames,
                                   size_t* bytes);

/* rehyat_forward with caller-provided device scratch (>= the size above,
 * 256-byte aligned); allocates nothing.  The workspace is overwritten. */
int rehyat_forward_ws(const void* q, const void* k, const void* v,
                      int B, int H, int F, int S_tok, int d,
                      int chunk_frames, int overlap_frames,
                      void* out, void* workspace, size_t workspace_bytes,
                      void* stream);

/* The two stages of rehyat_forward_ws, callable separately (same kernels):
 *   states:    phi(K), per-segment phi(K)^T V and sum phi(K), exclusive scan
 *              over chunks -> the state S_t, z_t entering each chunk, written
 *              into the workspace;
 *   attention: the fused per-chunk kernel (local softmax + phi(Q) S_t,
 *              phi(Q) z_t, joint normaliser), reading the states from the
 *              workspace filled by the states stage for the same shape. */
int rehyat_forward_states(const void* k, const void* v,
                          int B, int H, int F, int S_tok, int d,
                          int chunk_frames, int overlap_frames,
                          void* workspace, size_t workspace_bytes, void* stream);
int rehyat_forward_attention(const void* q, const void* k, const void* v,
                             int B, int H, int F, int S_tok, int d,
                             int chunk_frames, int overlap_frames,
                             void* out, void* workspace, size_t workspace_bytes,
                             void* stream);

/* Set modes of rehyat_forward_ex. */
#define REHYAT_SETS_CAUSAL 0        /* §3.3 recurrent sets: T^L_t = { j < lo_t } (rehyat_forward) */
#define REHYAT_SETS_BIDIRECTIONAL 1 /* §3.2 sets with overlap: T^L_t = T - T^S_t (earlier and later keys) */

/* Tensor layouts (q, k, v and out share one). */
#define REHYAT_LAYOUT_BHND 0  /* [B, H, N, d]: the layout of the entry points without a layout argument */
#define REHYAT_LAYOUT_BNHD 1  /* [B, N, H, d]: heads interleaved per token, as a DiT's
                                 attention projection writes them (no transpose needed) */

/* rehyat_forward with a choice of sets and of tensor layout.
 * REHYAT_SETS_BIDIRECTIONAL is the
 * non-causal variant (§3.2 sets with overlap; the causal vs non-causal
 * comparison of §5.3): chunk t's linear term covers every key outside its
 * softmax window [lo_t, min((t+1)N', N)), later keys included, so it has no
 * recurrent form.  workspace may be NULL (then stream-ordered scratch is
 * allocated and freed on `stream`), else it must hold
 * rehyat_forward_ex_workspace_bytes(..., sets) bytes, 256-byte aligned. */
int rehyat_forward_ex_workspace_bytes(int B, int H, int F, int S_tok, int d,
                                      int chunk_frames, int overlap_frames, int sets,
                                      size_t* bytes);
int rehyat_forward_ex(const void* q, const void* k, const void* v,
                      int B, int H, int F, int S_tok, int d,
                      int chunk_frames, int overlap_frames, int sets, int layout,
                      void* out, void* workspace, size_t workspace_bytes, void* stream);

/* Learned feature map ("ReHyAt", §4.3 Training specification and §7.1
 * Training Details: a two-layer MLP with degree-2 polynomial features,
 * separate maps for queries and keys; the §3.2 feature-map equation with
 * P = 2).  Per head h and row x (d wide):
 *   u   = W2[h] relu(W1[h] x + b1[h]) + b2[h]     (hidden width 2d)
 *   phi = [1 + elu(u[0:d]), (1 + elu(u[d:2d]))^2]  (2d wide, non-negative)
 * The paper fixes neither the hidden width nor the output non-linearity; this
 * reading keeps phi non-negative (§3.1) and gives about 2.4 M parameters per
 * block for 12 heads at d = 128 (the paper's figure).  With W1 = [I; -I],
 * W2 = [[I, -I]; [I, -I]] and zero biases it is the fixed phi.
 *   x   [B, H, N, d] or [B, N, H, d] (layout) bf16 device
 *   W1  [H, 2d, d] bf16, b1 [H, 2d] fp32, W2 [H, 2d, 2d] bf16, b2 [H, 2d] fp32
 *   phi [B, H, N, 2d] bf16 device, written (caller-owned, 16-byte aligned)
 * Tensor cores: both GEMMs accumulate in fp32; relu(W1 x + b1) is rounded
 * to bf16 before the second GEMM and phi to bf16 on output.  d is 64 or
 * 128.  Returns REHYAT_EINVAL for null / misaligned pointers or bad sizes. */
int rehyat_phi_mlp(const void* x, int B, int H, int N, int d, int layout,
                   const void* W1, const float* b1, const void* W2, const float* b2,
                   void* phi, void* stream);

/* rehyat_forward_ex with precomputed feature maps: phi_q, phi_k are
 * [B, H, N, 2d] bf16 device (any non-negative map, e.g. rehyat_phi_mlp's
 * output) used in place of the fixed phi in the linear term and the states:
 *   a^L = phi_q(q_i) S_t, n^L = phi_q(q_i) z_t, S_t = sum phi_k(k_j) v_j^T,
 *   z_t = sum phi_k(k_j) over T^L_t.  Workspace as rehyat_forward_ex (same
 *   size query).  q, k, v, out in `layout`; phi_q / phi_k always [B,H,N,2d]. */
int rehyat_forward_phi(const void* q, const void* k, const void* v,
                       const void* phi_q, const void* phi_k,
                       int B, int H, int F, int S_tok, int d,
                       int chunk_frames, int overlap_frames, int sets, int layout,
                       void* out, void* workspace, size_t workspace_bytes, void* stream);

/* The whole hybrid attention with learned feature maps: rehyat_phi_mlp of q
 * (weights Wq1, bq1, Wq2, bq2) and of k (Wk1, bk1, Wk2, bk2) in one launch
 * into the workspace, then rehyat_forward_phi.  Weight shapes as
 * rehyat_phi_mlp.  workspace may be NULL (stream-ordered scratch), else it
 * holds rehyat_forward_mlp_workspace_bytes(...) bytes, 256-byte aligned. */
int rehyat_forward_mlp_workspace_bytes(int B, int H, int F, int S_tok, int d,
                                       int chunk_frames, int overlap_frames, int sets,
                                       size_t* bytes);
int rehyat_forward_mlp(const void* q, const void* k, const void* v,
                       const void* Wq1, const float* bq1, const void* Wq2, const float* bq2,
                       const void* Wk1, const float* bk1, const void* Wk2, const float* bk2,
                       int B, int H, int F, int S_tok, int d,
                       int chunk_frames, int overlap_frames, int sets, int layout,
                       void* out, void* workspace, size_t workspace_bytes, void* stream);

/* rehyat_step (one chunk of the §3.3 recurrent form) with a tensor layout
 * and an optional caller workspace.
 *   layout  REHYAT_LAYOUT_BHND: q_c / out_c [B, H, Lq, d], k_c / v_c
 *           [B, H, Lk, d]; REHYAT_LAYOUT_BNHD: [B, Lq, H, d] / [B, Lk, H, d]
 *           (Lq = q_frames * S_tok, Lk = (ctx_frames + q_frames) * S_tok);
 *           all bf16 device, caller-owned, 16-byte aligned.  The state is
 *           always [B, H, 2d, d] / [B, H, 2d] fp32, updated in place.
 *   workspace  NULL: stream-ordered scratch allocated and freed on `stream`;
 *           else rehyat_step_workspace_bytes(...) bytes, 256-byte aligned.
 * Frame bookkeeping, results and asynchrony as rehyat_step: the output is
 * the [B, H, Lq, d] step's output in the chosen layout, bit for bit.
 * Returns REHYAT_EINVAL for an unknown layout, null / misaligned pointers or
 * bad sizes, REHYAT_ENOMEM for a workspace smaller than required; nothing is
 * launched after a validation failure. */
int rehyat_step_ex(const void* q_c, const void* k_c, const void* v_c,
                   float* state_S, float* state_z, void* out_c,
                   int B, int H, int S_tok, int d,
                   int q_frames, int ctx_frames, int evict_frames, int layout,
                   void* workspace, size_t workspace_bytes, void* stream);

/* rehyat_step with precomputed feature maps (e.g. rehyat_phi_mlp of the
 * chunk's q and of its window's k): phi_q_c [B, H, Lq, 2d] bf16 replaces the
 * fixed phi of q_c in the linear term, phi_k_c [B, H, Lk, 2d] bf16 that of
 * k_c when the first evict_frames * S_tok window keys are folded into the
 * state (only those rows are read).  Other arguments, the state update and
 * the frame bookkeeping as rehyat_step; workspace may be NULL (stream-ordered
 * scratch), else it holds rehyat_step_workspace_bytes(...) bytes, 256-byte
 * aligned. */
int rehyat_step_phi(const void* q_c, const void* k_c, const void* v_c,
                    const void* phi_q_c, const void* phi_k_c,
                    float* state_S, float* state_z, void* out_c,
                    int B, int H, int S_tok, int d,
                    int q_frames, int ctx_frames, int evict_frames,
                    void* workspace, size_t workspace_bytes, void* stream);

/* rehyat_forward_ex on HOST buffers: copies q, k, v (host, ideally
 * page-locked) into the device workspace, runs the forward, and copies the
 * result back into out_host, all enqueued on `stream` (asynchronous for
 * page-locked host memory: the result is in out_host once the stream has
 * reached this point; pageable memory makes the copies synchronous).
 * Keys and values are copied first, so the copy of q can overlap nothing but
 * is ready before the attention stage.  The workspace (device, 256-byte
 * aligned, caller-owned, rehyat_forward_host_workspace_bytes(...) bytes)
 * holds the device copies of q, k, v, out and the forward's scratch; callers
 * that alternate two workspaces on two streams overlap one call's copies with
 * another's kernels.  Host tensors in `layout`, [B, H, N, d] or [B, N, H, d]
 * bf16.  Returns REHYAT_ECUDA if a copy cannot be enqueued. */
int rehyat_forward_host_workspace_bytes(int B, int H, int F, int S_tok, int d,
                                        int chunk_frames, int overlap_frames, int sets,
                                        size_t* bytes);
int rehyat_forward_host(const void* q_host, const void* k_host, const void* v_host,
                        int B, int H, int F, int S_tok, int d,
                        int chunk_frames, int overlap_frames, int sets, int layout,
                        void* out_host, void* workspace, size_t workspace_bytes, void* stream);

/* fp32 forward (SIMT fp32 throughout, accurate exp) over the §3.3 causal
 * sets, [B, H, N, d] float tensors.  Meant for small problems and
 * tight-tolerance checks; any size is legal. */
int rehyat_forward_f32(const float* q, const float* k, const float* v,
                       int B, int H, int F, int S_tok, int d,
                       int chunk_frames, int overlap_frames,
                       float* out, void* stream);

/* fp32 counterparts of the learned-feature calls, for tight-tolerance checks:
 *   rehyat_phi_mlp_f32: the feature map of rehyat_phi_mlp in fp32 (no bf16
 *     rounding of the hidden layer or of phi); x [B, H, N, d], W1 [H, 2d, d],
 *     b1 [H, 2d], W2 [H, 2d, 2d], b2 [H, 2d] float, phi [B, H, N, 2d] float.
 *   rehyat_forward_phi_f32: rehyat_forward_f32 with precomputed features
 *     phi_q, phi_k [B, H, N, 2d] float in place of the fixed phi. */
int rehyat_phi_mlp_f32(const float* x, int B, int H, int N, int d,
                       const float* W1, const float* b1, const float* W2, const float* b2,
                       float* phi, void* stream);
int rehyat_forward_phi_f32(const float* q, const float* k, const float* v,
                           const float* phi_q, const float* phi_k,
                           int B, int H, int F, int S_tok, int d,
                           int chunk_frames, int overlap_frames,
                           float* out, void* stream);

/* Diagnostic form of rehyat_forward: runs the same fused tensor-core kernel
 * but writes the unnormalised terms of the §3.2 joint normaliser instead of
 * their ratio, all fp32, scaled by exp(-M):
 *   aS [B,H,N,d] = sum_{T^S} exp(s - M) v      nS [B,H,N] = sum_{T^S} exp(s - M)
 *   aL [B,H,N,d] = exp(-M) phi(q) S_t          nL [B,H,N] = exp(-M) phi(q) z_t
 *   M  [B,H,N]   = the shift used (natural log units), s = q.k/sqrt(d).
 * y = (aS + aL) / (nS + nL).  aL (and nL) are 0 where T^L_t is empty. */
int rehyat_forward_parts(const void* q, const void* k, const void* v,
                         int B, int H, int F, int S_tok, int d,
                         int chunk_frames, int overlap_frames,
                         float* aS, float* nS, float* aL, float* nL, float* M,
                         void* stream);

/* States entering each chunk, exported for inspection (bf16 inputs,
 * tensor-core phi(K)^T V, fp32 scan):  S [B,H,n_chunks,2d,d] fp32 (device,
 * caller-owned, 16-byte aligned), z [B,H,n_chunks,2d] fp32 (device,
 * caller-owned) with n_chunks = ceil(F / chunk_frames);
 * S_t = sum_{j < lo_t} phi(k_j) v_j^T, z_t = sum_{j < lo_t} phi(k_j).
 * Returns REHYAT_EINVAL for null or misaligned pointers or bad sizes. */
int rehyat_chunk_states(const void* k, const void* v,
                        int B, int H, int F, int S_tok, int d,
                        int chunk_frames, int overlap_frames,
                        float* S, float* z, void* stream);

/* rehyat_forward for callers that cannot allocate device memory during a
 * call (no counterpart in the paper: it is a deployment variant).  Examples:
 * a serving process that reserves all GPU memory at start-up and forbids
 * later allocation, because cudaMalloc may synchronise the device and has
 * unbounded latency; a plugin whose host framework owns the allocator and
 * exposes no scratch hook.  The caller still passes q, k, v and out as for
 * rehyat_forward; the scratch comes from a fixed array of
 * REHYAT_NOALLOC_SCRATCH_BYTES inside the library, which every GPU that
 * loads the library holds until the process exits.
 *   - Allocates nothing: no cudaMalloc / cudaMallocAsync / cudaFree.
 *   - When the default scratch layout does not fit, the key segments are
 *     summed in fewer pieces (fewer CTAs, same result up to fp32 rounding
 *     order); a problem that does not fit even then returns REHYAT_ENOMEM
 *     before launching anything (1.3B-480p needs ~30 MB and fits).
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current); make that first call
 *     before any stream capture.  Later calls made outside stream capture
 *     look it up again, so after a cudaDeviceReset the next ordinary call
 *     uses the reloaded array; calls recorded into a stream capture use the
 *     address of the last lookup on that device.
 *   - All calls on a device share the one array: calls whose kernels overlap
 *     on the GPU (different streams, no ordering) race and corrupt each
 *     other; order them.  Each call writes every scratch byte it reads. */
#define REHYAT_NOALLOC_SCRATCH_BYTES (32u << 20)
int rehyat_forward_noalloc(const void* q, const void* k, const void* v,
                           int B, int H, int F, int S_tok, int d,
                           int chunk_frames, int overlap_frames,
                           void* out, void* stream);

/* ---------------------------------------------------------------------- *
 * Recurrent form (§3.3 chunk-wise RNN), one chunk per call.               *
 * ---------------------------------------------------------------------- */

/* One chunk of the recurrent form with a constant-size state.
 *   q_c: [B,H,q_frames*S_tok,d]   the chunk's queries.
 *   k_c, v_c: [B,H,(ctx_frames+q_frames)*S_tok,d]  its whole softmax window:
 *        ctx_frames overlap frames followed by the chunk's own frames.
 *   state_S: [B,H,2d,d] fp32, state_z: [B,H,2d] fp32: the linear state of
 *        every key before the window (caller-owned; zero before chunk 0),
 *        updated IN PLACE: after the attention, the first evict_frames frames
 *        of k_c/v_c are folded in (S += phi(K)^T V, z += sum phi(K)).
 *   out_c: [B,H,q_frames*S_tok,d].
 * For chunk t of a video with window start w_t = max(t*T_c - T_o, 0):
 *   ctx_frames = t*T_c - w_t, q_frames = min(T_c, F - t*T_c),
 *   evict_frames = w_{t+1} - w_t   (w_{t+1} clipped to the window end).
 * 0 <= evict_frames <= ctx_frames + q_frames.  bf16 in, fp32 state. */
int rehyat_step(const void* q_c, const void* k_c, const void* v_c,
                float* state_S, float* state_z, void* out_c,
                int B, int H, int S_tok, int d,
                int q_frames, int ctx_frames, int evict_frames, void* stream);

/* Device scratch bytes one rehyat_step call of this shape needs (partial
 * states of the evicted keys and the state's bf16 hi/lo split); written to
 * *bytes.  Validates the arguments as rehyat_step does (REHYAT_EINVAL,
 * REHYAT_EUNSUPPORTED); launches nothing. */
int rehyat_step_workspace_bytes(int B, int H, int S_tok, int d,
                                int q_frames, int ctx_frames, int evict_frames,
                                size_t* bytes);

/* rehyat_step with caller-provided scratch; allocates nothing. */
int rehyat_step_ws(const void* q_c, const void* k_c, const void* v_c,
                   float* state_S, float* state_z, void* out_c,
                   int B, int H, int S_tok, int d,
                   int q_frames, int ctx_frames, int evict_frames,
                   void* workspace, size_t workspace_bytes, void* stream);

/* fp32 step (SIMT), same contract with float tensors. */
int rehyat_step_f32(const float* q_c, const float* k_c, const float* v_c,
                    float* state_S, float* state_z, float* out_c,
                    int B, int H, int S_tok, int d,
                    int q_frames, int ctx_frames, int evict_frames, void* stream);

/* ---------------------------------------------------------------------- *
 * Feature map and device status.                                          *
 * ---------------------------------------------------------------------- */

#define REHYAT_DTYPE_BF16 0
#define REHYAT_DTYPE_F32 1

/* §3.2 feature map phi(x) = [psi(x), psi(x)^2], psi = 1 + elu (§3.1),
 * row-wise: x [rows, d] -> y [rows, 2d], any d >= 1.  dtype codes
 * REHYAT_DTYPE_*; x, y device memory aligned to their element size.
 * Returns REHYAT_EINVAL for null / misaligned pointers, an unknown dtype or
 * bad sizes. */
int rehyat_phi(const void* x, int x_dtype, void* y, int y_dtype,
               int64_t rows, int d, void* stream);

/* Diagnostic for the failure path: launches one warp that waits on a
 * barrier nothing ever completes.  The wait is bounded like every device
 * wait in this library (2 s of GPU time); it then records the timeout in the
 * device error word and the kernel returns, so rehyat_device_status()
 * reports REHYAT_ETIMEOUT once and later calls run normally.  gave_up: NULL
 * or one device int, set to 1 when the wait gave up (0 had it completed).
 * Returns REHYAT_ECUDA if the launch fails. */
int rehyat_wait_probe(int* gave_up, void* stream);

/* Synchronises the current device and reports whether any kernel of this
 * library recorded a device-side error since the last call (REHYAT_ETIMEOUT
 * when a bounded wait ran out), then clears the record.  *detail (optional)
 * receives the raw error word (0 when clean). */
int rehyat_device_status(unsigned int* detail);

#ifdef __cplusplus
}
#endif

#endif /* REHYAT_H */
