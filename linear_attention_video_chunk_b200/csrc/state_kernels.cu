// state_kernels.cu -- the memory-bound SIMT steps around the chunk states
// of "ReHyAt: Recurrent Hybrid Attention for Video Diffusion Transformers":
// the exclusive scan over chunks of the per-segment sums (§3.1 caching, §3.3
// sets), its bidirectional counterpart (§3.2 sets with overlap), the
// recurrent form's state update (§3.3), and the fp32 -> bf16 hi/lo split the
// tensor-core epilogue reads.
#include <cstdint>

#include <cuda_bf16.h>

#include "kernels.cuh"

namespace rehyat {
namespace {

// ============================================================================
// Scan / accumulate / split (SIMT, memory-bound)
// ============================================================================
// One thread per state entry (bh, e, c) with c == D meaning z: walks the
// chunks in order, writing the exclusive prefix, then adding segment t.
__global__ void state_scan_kernel(const float* __restrict__ pS, const float* __restrict__ pz, int BH,
                                  int n_seg, int nsplit, int nc, int D, __nv_bfloat16* hi,
                                  __nv_bfloat16* lo, float* Sf, float* zt) {
  const int W = D + 1;
  const long long total = static_cast<long long>(BH) * 2 * D * W;
  for (long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int c = static_cast<int>(idx % W);
    const int e = static_cast<int>((idx / W) % (2 * D));
    const int bh = static_cast<int>(idx / (static_cast<long long>(W) * 2 * D));
    float acc = 0.f;
    for (int t = 0; t < nc; ++t) {
      const size_t so = ((static_cast<size_t>(bh) * nc + t) * 2 * D + e);
      if (c == D) {
        zt[so] = acc;
      } else if (hi != nullptr) {
        const __nv_bfloat16 h = __float2bfloat16_rn(acc);
        hi[so * D + c] = h;
        lo[so * D + c] = __float2bfloat16_rn(acc - __bfloat162float(h));
      } else {
        Sf[so * D + c] = acc;
      }
      if (t < n_seg) {
        for (int pp = 0; pp < nsplit; ++pp) {
          const size_t po = (static_cast<size_t>(bh) * n_seg + t) * nsplit + pp;
          acc += (c == D) ? pz[po * 2 * D + e] : pS[(po * 2 * D + e) * D + c];
        }
      }
    }
  }
}

// Bidirectional sets: segments are frames; for chunk t with window frames
// [lo_f, hi_f) the state is sum over frames < lo_f plus frames >= hi_f.  One
// thread per state entry walks the frames twice (total, then the two
// monotone prefix pointers), in a fixed order.
__global__ void state_scan_bidir_kernel(const float* __restrict__ pS, const float* __restrict__ pz, int BH,
                                        int F, int nsplit, int nc, int D, int Tc, int To, __nv_bfloat16* hi,
                                        __nv_bfloat16* lo, float* Sf, float* zt) {
  const int W = D + 1;
  const long long total = static_cast<long long>(BH) * 2 * D * W;
  for (long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int c = static_cast<int>(idx % W);
    const int e = static_cast<int>((idx / W) % (2 * D));
    const int bh = static_cast<int>(idx / (static_cast<long long>(W) * 2 * D));
    auto frame = [&](int f) {
      float acc = 0.f;
      for (int pp = 0; pp < nsplit; ++pp) {
        const size_t po = (static_cast<size_t>(bh) * F + f) * nsplit + pp;
        acc += (c == D) ? pz[po * 2 * D + e] : pS[(po * 2 * D + e) * D + c];
      }
      return acc;
    };
    float tot = 0.f;
    for (int f = 0; f < F; ++f) tot += frame(f);
    float p_lo = 0.f, p_hi = 0.f;  // prefix sums up to lo_f and hi_f
    int f_lo = 0, f_hi = 0;
    for (int t = 0; t < nc; ++t) {
      const int lo_f = imax(t * Tc - To, 0), hi_f = imin((t + 1) * Tc, F);
      for (; f_lo < lo_f; ++f_lo) p_lo += frame(f_lo);
      for (; f_hi < hi_f; ++f_hi) p_hi += frame(f_hi);
      const float acc = p_lo + (tot - p_hi);
      const size_t so = ((static_cast<size_t>(bh) * nc + t) * 2 * D + e);
      if (c == D) {
        zt[so] = acc;
      } else if (hi != nullptr) {
        const __nv_bfloat16 h = __float2bfloat16_rn(acc);
        hi[so * D + c] = h;
        lo[so * D + c] = __float2bfloat16_rn(acc - __bfloat162float(h));
      } else {
        Sf[so * D + c] = acc;
      }
    }
  }
}

__global__ void state_accumulate_kernel(const float* __restrict__ pS, const float* __restrict__ pz, int BH,
                                        int nsplit, int D, float* S, float* z) {
  // In the recurrent step this kernel follows the fold of evicted keys with
  // a programmatic dependency: wait until that fold (and so the attention
  // before it, which reads z) has completed.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int W = D + 1;
  const long long total = static_cast<long long>(BH) * 2 * D * W;
  for (long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int c = static_cast<int>(idx % W);
    const int e = static_cast<int>((idx / W) % (2 * D));
    const int bh = static_cast<int>(idx / (static_cast<long long>(W) * 2 * D));
    float acc = 0.f;
    for (int pp = 0; pp < nsplit; ++pp) {
      const size_t po = static_cast<size_t>(bh) * nsplit + pp;
      acc += (c == D) ? pz[po * 2 * D + e] : pS[(po * 2 * D + e) * D + c];
    }
    if (c == D)
      z[static_cast<size_t>(bh) * 2 * D + e] += acc;
    else
      S[(static_cast<size_t>(bh) * 2 * D + e) * D + c] += acc;
  }
}

__global__ void state_split_kernel(const float* __restrict__ S, long long n, __nv_bfloat16* hi,
                                   __nv_bfloat16* lo) {
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const float x = S[i];
    const __nv_bfloat16 h = __float2bfloat16_rn(x);
    hi[i] = h;
    lo[i] = __float2bfloat16_rn(x - __bfloat162float(h));
  }
}

int grid_for(long long n, int threads) {
  long long g = (n + threads - 1) / threads;
  if (g > 148LL * 16) g = 148LL * 16;
  return static_cast<int>(g < 1 ? 1 : g);
}

}  // namespace

cudaError_t launch_state_scan(const float* part_S, const float* part_z, int BH, int n_seg, int nsplit,
                              int n_chunks, int D, __nv_bfloat16* hi, __nv_bfloat16* lo, float* Sf,
                              float* zt, cudaStream_t s) {
  const long long n = static_cast<long long>(BH) * 2 * D * (D + 1);
  state_scan_kernel<<<grid_for(n, 256), 256, 0, s>>>(part_S, part_z, BH, n_seg, nsplit, n_chunks, D, hi, lo,
                                                      Sf, zt);
  return cudaGetLastError();
}

cudaError_t launch_state_scan_bidir(const float* part_S, const float* part_z, int BH, int F, int nsplit,
                                    int n_chunks, int D, int Tc, int To, __nv_bfloat16* hi, __nv_bfloat16* lo,
                                    float* Sf, float* zt, cudaStream_t s) {
  const long long n = static_cast<long long>(BH) * 2 * D * (D + 1);
  state_scan_bidir_kernel<<<grid_for(n, 256), 256, 0, s>>>(part_S, part_z, BH, F, nsplit, n_chunks, D, Tc, To, hi,
                                                            lo, Sf, zt);
  return cudaGetLastError();
}

cudaError_t launch_state_accumulate(const float* part_S, const float* part_z, int BH, int nsplit, int D,
                                    float* state_S, float* state_z, cudaStream_t s, bool pdl) {
  const long long n = static_cast<long long>(BH) * 2 * D * (D + 1);
  return launch_k(state_accumulate_kernel, dim3(grid_for(n, 256)), dim3(256), 0, s, pdl, part_S, part_z, BH, nsplit,
                  D, state_S, state_z);
}

cudaError_t launch_state_split(const float* S, long long n, __nv_bfloat16* hi, __nv_bfloat16* lo,
                               cudaStream_t s) {
  state_split_kernel<<<grid_for(n, 256), 256, 0, s>>>(S, n, hi, lo);
  return cudaGetLastError();
}

}  // namespace rehyat
