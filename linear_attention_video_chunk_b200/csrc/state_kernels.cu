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

// The two key-window halves of every split unit of the fused attention:
// one thread per (split unit, query tile, row, group of 8 columns).  The
// partial rows hold O (unnormalised, scaled by 2^-m), the denominator L on
// the same scale, and the shift m (log2 units); the halves combine on the
// larger shift.  Launched with a programmatic dependency right behind the
// attention, so it waits for it first.
__global__ void split_merge_kernel(const float* __restrict__ part, int n_split, int split_begin, int BH, int H,
                                   int N_q, int D, __nv_bfloat16* __restrict__ out, long long o_sb, long long o_sh,
                                   long long o_sr) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int G8 = D / 8;
  const long long total = static_cast<long long>(n_split) * 2 * 128 * G8;
  const size_t W = static_cast<size_t>(D) + 4;
  for (long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int g = static_cast<int>(idx % G8);
    const long long rr = idx / G8;
    const int r = static_cast<int>(rr % 128);
    const int X = static_cast<int>((rr / 128) % 2);
    const int i = static_cast<int>(rr / 256);
    const int o = split_begin + i;  // pair-major unit number
    const int pair = o / BH, bh = o % BH;
    const int qrow = pair * 256 + X * 128 + r;
    if (qrow >= N_q) continue;
    const float* e0 = part + ((static_cast<size_t>(i * 2 + 0) * 2 + X) * 128 + r) * W;
    const float* e1 = part + ((static_cast<size_t>(i * 2 + 1) * 2 + X) * 128 + r) * W;
    const float m0 = e0[D + 1], m1 = e1[D + 1];
    const float M = fmaxf(m0, m1);
    const float w0 = exp2f(m0 - M), w1 = exp2f(m1 - M);
    const float inv = 1.f / (e0[D] * w0 + e1[D] * w1);
    const float4 a0 = reinterpret_cast<const float4*>(e0 + 8 * g)[0], b0 = reinterpret_cast<const float4*>(e0 + 8 * g)[1];
    const float4 a1 = reinterpret_cast<const float4*>(e1 + 8 * g)[0], b1 = reinterpret_cast<const float4*>(e1 + 8 * g)[1];
    const float y[8] = {a0.x * w0 + a1.x * w1, a0.y * w0 + a1.y * w1, a0.z * w0 + a1.z * w1, a0.w * w0 + a1.w * w1,
                        b0.x * w0 + b1.x * w1, b0.y * w0 + b1.y * w1, b0.z * w0 + b1.z * w1, b0.w * w0 + b1.w * w1};
    uint32_t pk[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      __nv_bfloat162 h2 = __floats2bfloat162_rn(y[2 * c] * inv, y[2 * c + 1] * inv);
      pk[c] = *reinterpret_cast<uint32_t*>(&h2);
    }
    *reinterpret_cast<uint4*>(out + (bh / H) * o_sb + (bh % H) * o_sh + qrow * o_sr + 8 * g) =
        make_uint4(pk[0], pk[1], pk[2], pk[3]);
  }
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

cudaError_t launch_split_merge(const float* part, int n_split, int split_begin, int BH, int H, int N_q, int D,
                               __nv_bfloat16* out, long long o_sb, long long o_sh, long long o_sr, cudaStream_t s,
                               bool pdl) {
  if (n_split <= 0) return cudaSuccess;
  const long long n = static_cast<long long>(n_split) * 2 * 128 * (D / 8);
  return launch_k(split_merge_kernel, dim3(grid_for(n, 256)), dim3(256), 0, s, pdl, part, n_split, split_begin, BH,
                  H, N_q, D, out, o_sb, o_sh, o_sr);
}

cudaError_t launch_state_split(const float* S, long long n, __nv_bfloat16* hi, __nv_bfloat16* lo,
                               cudaStream_t s) {
  state_split_kernel<<<grid_for(n, 256), 256, 0, s>>>(S, n, hi, lo);
  return cudaGetLastError();
}

}  // namespace rehyat
