// mlp.cuh -- parameter block and launcher of the learned feature-map kernel
// (internal to librehyat).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace rehyat {

// Learned feature map (two-layer MLP, degree-2 polynomial features) on the
// tensor cores: phi[row] = [psi_1, psi_2^2] of u = W2 relu(W1 x + b1) + b2,
// psi = 1 + elu.  Up to two maps (phi_q of q, phi_k of k) per launch; one CTA
// per (map, bh, row group) walks that group's 128-row tiles.
struct MlpParams {
  CUtensorMap tm_x[2];    // 4-D {D, N, H, B} bf16, box {64, 128, 1, 1}
  CUtensorMap tm_w1[2];   // [H, 2D, D] bf16, box {64, 2D, 1}
  CUtensorMap tm_w2[2];   // [H, 2D, 2D] bf16, box {64, 2D, 1}
  const float* b1[2];     // [H, 2D]
  const float* b2[2];     // [H, 2D]
  __nv_bfloat16* phi[2];  // [BH, N, 2D]
  int N, H, BH, groups;
  unsigned long long* trace;  // clock64 stamps, only with -DREHYAT_TRACE (else unused)
};

cudaError_t launch_phi_mlp(int D, const MlpParams& p, int n_maps, cudaStream_t s);

}  // namespace rehyat
