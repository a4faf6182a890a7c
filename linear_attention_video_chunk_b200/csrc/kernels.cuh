// kernels.cuh -- kernel parameter blocks and launchers (internal to librehyat).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <mutex>
#include <set>
#include <utility>

#include "geom.cuh"

namespace rehyat {

// Fused per-chunk hybrid attention (tensor cores).  One CTA = one "unit":
// up to two 128-row query tiles of one chunk of one (b,h).
struct AttnParams {
  // q / k / v maps are 4-D {D, rows, H, B} with per-dimension strides (any of
  // the [B,H,N,d] or [B,N,H,d] layouts), box {64, 128, 1, 1}, 128B swizzle.
  CUtensorMap tm_q;
  CUtensorMap tm_k;
  CUtensorMap tm_v;
  CUtensorMap tm_hi;  // [BH * state_mul, 2D, D] bf16: high part of S_t
  CUtensorMap tm_lo;  // same: S_t - hi (rounded to bf16)
  ChunkGeom g;
  int BH;
  int H;              // heads: bh = b * H + h
  int pairs;          // units per (bh, chunk)
  int state_mul;      // state tile z-coordinate = bh * state_mul + (g.step ? 0 : t)
  float scale_log2;   // log2(e) / sqrt(D)
  const float* z;     // z_t (fp32); entry e of (bh, t) at z[bh*z_bh + t*z_t + e]
  long long z_bh, z_t;
  __nv_bfloat16* out; // element (b, h, row, c) at out[b*o_sb + h*o_sh + row*o_sr + c]
  long long o_sb, o_sh, o_sr;
  float* aS;          // diagnostic parts, [BH, N_q, D] / [BH, N_q] (PARTS kernels only)
  float* nS;
  float* aL;
  float* nL;
  float* Mo;
  const __nv_bfloat16* phi_q;  // [BH, N_q, 2D] precomputed phi(q) (feature-map variant only)
  unsigned long long* trace;   // clock64 stamps, only with -DREHYAT_TRACE (else unused)
  // Units are numbered o = pair * BH + bh when pair_major (one chunk, the
  // recurrent step), else o = (chunk order * BH + bh) * pairs + pair.  The
  // n_split units o in [split_begin, split_begin + n_split) run as two CTAs
  // each, over the first and the second half of the key window, and write
  // partial rows instead of the output: launch index u runs o = u below
  // split_begin, then the two halves of each split unit, then o = u - n_split.
  int pair_major;
  int split_begin;
  int n_split;
  float* part;        // [n_split, 2 halves, 2 query tiles, 128 rows, D + 4] fp32: O, denominator, shift, 2 pad
};

// phi(K)^T V and sum phi(K) over key segments (tensor cores).  One CTA =
// one piece of one segment of one (b,h).
struct StateParams {
  CUtensorMap tm_k;   // 4-D {D, rows, H, B} bf16, box {64, 64, 1, 1}
  CUtensorMap tm_v;
  CUtensorMap tm_phik; // 4-D {2D, N, H, B} bf16 box {64, 64, 1, 1} (feature-map variant only)
  SegGeom sg;
  int BH;
  int H;
  float* part_S;      // [BH, n_seg, nsplit, 2D, D] fp32
  float* part_z;      // [BH, n_seg, nsplit, 2D] fp32
};

// fp32 SIMT paths
struct AttnF32Params {
  ChunkGeom g;
  int BH, D;
  const float* q;     // [BH, N_q, D]
  const float* k;     // [BH, N_k, D]
  const float* v;
  const float* S;     // S_t at S[bh*S_bh + t*S_t] ([2D, D] row-major)
  long long S_bh, S_t;
  const float* z;     // z_t at z[bh*z_bh + t*z_t]
  long long z_bh, z_t;
  float* out;         // [BH, N_q, D]
  const float* phi_q; // optional [BH, N_q, 2D] precomputed phi(q) (null: the fixed phi of q)
};

struct StateF32Params {
  SegGeom sg;         // nsplit must be 1
  int BH, D;
  const float* k;
  const float* v;
  float* part_S;      // [BH, n_seg, 1, 2D, D]
  float* part_z;
  const float* phi_k; // optional [BH, N_k, 2D] precomputed phi(k) (null: the fixed phi of k)
};

// One-time per-device setup of a kernel before its first launch: allow
// `smem` bytes of dynamic shared memory and, when need_regs > 0, check that
// it compiled to exactly need_regs registers a thread.  Later launches skip
// both calls, so launches can be captured into CUDA graphs.
inline cudaError_t prepare_kernel_once(const void* func, int smem, int need_regs) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static std::mutex mu;
  static std::set<std::pair<const void*, int>> done;
  std::lock_guard<std::mutex> lock(mu);
  if (done.count({func, dev})) return cudaSuccess;
  if (need_regs > 0) {
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, func);
    if (e != cudaSuccess) return e;
    if (fa.numRegs != need_regs) return cudaErrorInvalidConfiguration;
  }
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e == cudaSuccess) done.insert({func, dev});
  return e;
}

// Launch `k` on stream s; with pdl the launch carries a programmatic
// dependency on the previous kernel in the stream, so its CTAs may be
// scheduled before that kernel has finished (the kernel itself waits, with
// griddepcontrol.wait, before touching what the previous kernel writes).
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*k)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, bool pdl,
                     Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, k, std::forward<Args>(args)...);
}

// Shared-memory bytes each tensor-core kernel needs (dynamic).
int attn_smem_bytes(int D);
int state_smem_bytes(int D);

cudaError_t launch_attention(int D, bool parts, const AttnParams& p, int n_units, cudaStream_t s, bool pdl = false);
cudaError_t launch_chunk_state(int D, const StateParams& p, int n_ctas, cudaStream_t s, bool pdl = false);
// Variants reading precomputed feature maps: phi(K) through p.tm_phik (the
// states) and phi(Q) rows from p.phi_q (the attention epilogue).
cudaError_t launch_attention_phi(int D, const AttnParams& p, int n_units, cudaStream_t s, bool pdl = false);
cudaError_t launch_chunk_state_phi(int D, const StateParams& p, int n_ctas, cudaStream_t s, bool pdl = false);
// Exclusive prefix over segments (and sum over pieces): writes the state
// entering each chunk, either as bf16 hi/lo (hi, lo non-null) or fp32 (Sf).
cudaError_t launch_state_scan(const float* part_S, const float* part_z, int BH, int n_seg,
                              int nsplit, int n_chunks, int D, __nv_bfloat16* hi,
                              __nv_bfloat16* lo, float* Sf, float* zt, cudaStream_t s);
// Bidirectional sets: per-frame partials -> prefix(lo_t) + suffix(hi_t).
cudaError_t launch_state_scan_bidir(const float* part_S, const float* part_z, int BH, int F, int nsplit,
                                    int n_chunks, int D, int Tc, int To, __nv_bfloat16* hi, __nv_bfloat16* lo,
                                    float* Sf, float* zt, cudaStream_t s);
// Combine the two key-window halves of every split unit (AttnParams): out =
// (O0 2^(m0-M) + O1 2^(m1-M)) / (L0 2^(m0-M) + L1 2^(m1-M)), M = max(m0, m1).
cudaError_t launch_split_merge(const float* part, int n_split, int split_begin, int BH, int H, int N_q, int D,
                               __nv_bfloat16* out, long long o_sb, long long o_sh, long long o_sr, cudaStream_t s,
                               bool pdl);
// state_S/z += sum over pieces of one segment's partials.
cudaError_t launch_state_accumulate(const float* part_S, const float* part_z, int BH, int nsplit,
                                    int D, float* state_S, float* state_z, cudaStream_t s, bool pdl = false);
// fp32 state -> bf16 hi/lo pair.
cudaError_t launch_state_split(const float* S, long long n, __nv_bfloat16* hi, __nv_bfloat16* lo,
                               cudaStream_t s);

cudaError_t launch_attention_f32(const AttnF32Params& p, int n_chunks, cudaStream_t s);
cudaError_t launch_chunk_state_f32(const StateF32Params& p, cudaStream_t s);
cudaError_t launch_phi(const void* x, int x_f32, void* y, int y_f32, long long rows, int d,
                       cudaStream_t s);
// Learned feature map in fp32 SIMT: x [BH, N, d] (head = (row / N) % H),
// W1 [H, 2d, d], b1 [H, 2d], W2 [H, 2d, 2d], b2 [H, 2d] -> phi [BH, N, 2d].
cudaError_t launch_phi_mlp_f32(const float* x, long long rows, int N, int H, int d, const float* W1,
                               const float* b1, const float* W2, const float* b2, float* phi, cudaStream_t s);

}  // namespace rehyat
