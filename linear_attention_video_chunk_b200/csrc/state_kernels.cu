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
// The vector kernels below give each thread four consecutive state columns
// (one float4) of one row e of one (b,h); the thread holding columns 0..3
// also carries z[e].  Every pointer is 16-byte aligned and D % 4 == 0, so
// the float4 loads and 8-byte bf16 stores are aligned.
struct Row4 {
  int bh, e, c;  // c = first of the four columns
  bool z;        // this thread also carries z[e]
};
__device__ __forceinline__ Row4 row4(long long idx, int D) {
  // D is 64 or 128: D / 4 and 2D are powers of two (shifts, no division)
  const int lg = (D == 128) ? 5 : 4;  // log2(D / 4); log2(2D) = lg + 3
  Row4 r;
  r.c = 4 * static_cast<int>(idx & ((1 << lg) - 1));
  r.e = static_cast<int>((idx >> lg) & ((2 * D) - 1));
  r.bh = static_cast<int>(idx >> (2 * lg + 3));
  r.z = r.c == 0;
  return r;
}
__device__ __forceinline__ void add4(float4& a, const float4 b) {
  a.x += b.x;
  a.y += b.y;
  a.z += b.z;
  a.w += b.w;
}
// The state entering a chunk: fp32 (Sf) or the bf16 pair hi = bf16(S),
// lo = bf16(S - hi) the tensor-core epilogue reads.
__device__ __forceinline__ void put_state(size_t so, const Row4& r, int D, const float4 acc, float az,
                                          __nv_bfloat16* __restrict__ hi, __nv_bfloat16* __restrict__ lo,
                                          float* __restrict__ Sf, float* __restrict__ zt) {
  if (r.z) zt[so] = az;
  const size_t o = so * D + r.c;
  if (hi != nullptr) {
    const float v[4] = {acc.x, acc.y, acc.z, acc.w};
    __nv_bfloat16 h[4], l[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      h[i] = __float2bfloat16_rn(v[i]);
      l[i] = __float2bfloat16_rn(v[i] - __bfloat162float(h[i]));
    }
    *reinterpret_cast<uint2*>(hi + o) = *reinterpret_cast<const uint2*>(h);
    *reinterpret_cast<uint2*>(lo + o) = *reinterpret_cast<const uint2*>(l);
  } else {
    *reinterpret_cast<float4*>(Sf + o) = acc;
  }
}

// Exclusive scan over chunks: chunk t receives the sum of segments 0..t-1,
// each segment the sum of its pieces in piece order.  The (segment, piece)
// items are read eight at a time ahead of the sums (the loads do not depend
// on them; past the last item the index is clamped, so every load is valid).
__global__ void state_scan_kernel(const float* __restrict__ pS, const float* __restrict__ pz, int BH,
                                  int n_seg, int nsplit, int nc, int D, __nv_bfloat16* __restrict__ hi,
                                  __nv_bfloat16* __restrict__ lo, float* __restrict__ Sf, float* __restrict__ zt) {
  constexpr int PF = 8;
  const long long total = static_cast<long long>(BH) * 2 * D * (D / 4);
  const int n_items = n_seg * nsplit;  // per (b,h); the planner bounds BH * n_items by INT_MAX
  for (long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<long long>(gridDim.x) * blockDim.x) {
    const Row4 r = row4(idx, D);
    const size_t so0 = static_cast<size_t>(r.bh) * nc * 2 * D + r.e;  // (bh, t = 0, e)
    const size_t po0 = static_cast<size_t>(r.bh) * n_items;           // (bh, segment 0, piece 0)
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float az = 0.f;
    int t_next = 0;  // the next chunk whose state is still to be written
    int pp = 0;      // piece of the next item
    for (int j0 = 0; j0 < n_items; j0 += PF) {
      float4 v[PF];
      float vz[PF];
#pragma unroll
      for (int i = 0; i < PF; ++i) {
        const size_t po = po0 + static_cast<size_t>(imin(j0 + i, n_items - 1));
        v[i] = __ldg(reinterpret_cast<const float4*>(pS + (po * 2 * D + r.e) * D + r.c));
        vz[i] = r.z ? __ldg(pz + po * 2 * D + r.e) : 0.f;
      }
#pragma unroll
      for (int i = 0; i < PF; ++i) {
        if (j0 + i < n_items) {
          if (pp == 0)  // the first piece of segment t_next: chunk t_next's prefix is complete
            put_state(so0 + static_cast<size_t>(t_next++) * 2 * D, r, D, acc, az, hi, lo, Sf, zt);
          add4(acc, v[i]);
          az += vz[i];
          if (++pp == nsplit) pp = 0;
        }
      }
    }
    for (; t_next < nc; ++t_next) put_state(so0 + static_cast<size_t>(t_next) * 2 * D, r, D, acc, az, hi, lo, Sf, zt);
  }
}

// Bidirectional sets: segments are frames; for chunk t with window frames
// [lo_f, hi_f) the state is sum over frames < lo_f plus frames >= hi_f.  One
// thread per four state entries walks the frames twice (total, then the two
// monotone prefix pointers), in a fixed order.
__global__ void state_scan_bidir_kernel(const float* __restrict__ pS, const float* __restrict__ pz, int BH,
                                        int F, int nsplit, int nc, int D, int Tc, int To,
                                        __nv_bfloat16* __restrict__ hi, __nv_bfloat16* __restrict__ lo,
                                        float* __restrict__ Sf, float* __restrict__ zt) {
  const long long total = static_cast<long long>(BH) * 2 * D * (D / 4);
  for (long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<long long>(gridDim.x) * blockDim.x) {
    const Row4 r = row4(idx, D);
    auto frame = [&](int f, float& fz) {
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      fz = 0.f;
      for (int pp = 0; pp < nsplit; ++pp) {
        const size_t po = (static_cast<size_t>(r.bh) * F + f) * nsplit + pp;
        add4(acc, __ldg(reinterpret_cast<const float4*>(pS + (po * 2 * D + r.e) * D + r.c)));
        if (r.z) fz += __ldg(pz + po * 2 * D + r.e);
      }
      return acc;
    };
    float4 tot = make_float4(0.f, 0.f, 0.f, 0.f);
    float tz = 0.f, fz;
    for (int f = 0; f < F; ++f) {
      add4(tot, frame(f, fz));
      tz += fz;
    }
    float4 p_lo = make_float4(0.f, 0.f, 0.f, 0.f), p_hi = p_lo;  // prefix sums up to lo_f and hi_f
    float z_lo = 0.f, z_hi = 0.f;
    int f_lo = 0, f_hi = 0;
    for (int t = 0; t < nc; ++t) {
      const int lo_f = imax(t * Tc - To, 0), hi_f = imin((t + 1) * Tc, F);
      for (; f_lo < lo_f; ++f_lo) {
        add4(p_lo, frame(f_lo, fz));
        z_lo += fz;
      }
      for (; f_hi < hi_f; ++f_hi) {
        add4(p_hi, frame(f_hi, fz));
        z_hi += fz;
      }
      const float4 acc = make_float4(p_lo.x + (tot.x - p_hi.x), p_lo.y + (tot.y - p_hi.y), p_lo.z + (tot.z - p_hi.z),
                                     p_lo.w + (tot.w - p_hi.w));
      put_state(static_cast<size_t>(r.bh) * nc * 2 * D + static_cast<size_t>(t) * 2 * D + r.e, r, D, acc,
                z_lo + (tz - z_hi), hi, lo, Sf, zt);
    }
  }
}

__global__ void state_accumulate_kernel(const float* __restrict__ pS, const float* __restrict__ pz, int BH,
                                        int nsplit, int D, float* __restrict__ S, float* __restrict__ z) {
  // In the recurrent step this kernel follows the fold of evicted keys with
  // a programmatic dependency: wait until that fold (and so the attention
  // before it, which reads z) has completed.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const long long total = static_cast<long long>(BH) * 2 * D * (D / 4);
  for (long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<long long>(gridDim.x) * blockDim.x) {
    const Row4 r = row4(idx, D);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float az = 0.f;
    for (int pp = 0; pp < nsplit; ++pp) {
      const size_t po = static_cast<size_t>(r.bh) * nsplit + pp;
      add4(acc, __ldg(reinterpret_cast<const float4*>(pS + (po * 2 * D + r.e) * D + r.c)));
      if (r.z) az += __ldg(pz + po * 2 * D + r.e);
    }
    const size_t so = static_cast<size_t>(r.bh) * 2 * D + r.e;
    float4* dst = reinterpret_cast<float4*>(S + so * D + r.c);
    float4 cur = *dst;
    add4(cur, acc);
    *dst = cur;
    if (r.z) z[so] += az;
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
  const long long n = static_cast<long long>(BH) * 2 * D * (D / 4);
  state_scan_kernel<<<grid_for(n, 256), 256, 0, s>>>(part_S, part_z, BH, n_seg, nsplit, n_chunks, D, hi, lo,
                                                      Sf, zt);
  return cudaGetLastError();
}

cudaError_t launch_state_scan_bidir(const float* part_S, const float* part_z, int BH, int F, int nsplit,
                                    int n_chunks, int D, int Tc, int To, __nv_bfloat16* hi, __nv_bfloat16* lo,
                                    float* Sf, float* zt, cudaStream_t s) {
  const long long n = static_cast<long long>(BH) * 2 * D * (D / 4);
  state_scan_bidir_kernel<<<grid_for(n, 256), 256, 0, s>>>(part_S, part_z, BH, F, nsplit, n_chunks, D, Tc, To, hi,
                                                            lo, Sf, zt);
  return cudaGetLastError();
}

cudaError_t launch_state_accumulate(const float* part_S, const float* part_z, int BH, int nsplit, int D,
                                    float* state_S, float* state_z, cudaStream_t s, bool pdl) {
  const long long n = static_cast<long long>(BH) * 2 * D * (D / 4);
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
