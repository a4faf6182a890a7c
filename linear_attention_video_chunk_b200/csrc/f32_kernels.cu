// f32_kernels.cu -- fp32 SIMT kernels: the whole hybrid attention in fp32
// with accurate exp (for tight-tolerance checks and fp32 callers), and the
// standalone feature map.
//
// "ReHyAt: Recurrent Hybrid Attention for Video Diffusion Transformers":
//   §3.1 linear attention through the cached sums S = sum phi(k) v^T,
//        z = sum phi(k); phi non-negative, psi = 1 + elu;
//   §3.2 joint normaliser y = (a^S + a^L) / (n^S + n^L) and the polynomial
//        feature map phi = [psi, psi^2] (P = 2);
//   §3.3 recurrent sets (softmax window [lo_t, hi_t), linear set [0, lo_t)).
#include <cstdint>

#include "kernels.cuh"

namespace rehyat {
namespace {

constexpr uint32_t kFull = 0xffffffffu;

__device__ __forceinline__ float psi_f32(float x) { return x > 0.f ? x + 1.f : expf(x); }

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(kFull, x, o);
  return x;
}

// One warp per query row; lane owns columns lane + 32 i.  Exact online
// softmax over the window, the shift starting at 0 when the linear set is
// non-empty (so exp(-M) <= 1 multiplies the linear terms), then
// y = (acc + e^{-M} phi(q) S_t) / (l + e^{-M} phi(q) z_t).
template <int PER>
__global__ void __launch_bounds__(256) attn_f32_kernel(const AttnF32Params p) {
  constexpr int D = PER * 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.y, bh = blockIdx.z;
  int q0, q1, lo, hi;
  p.g.chunk(t, q0, q1, lo, hi);
  const int row = q0 + blockIdx.x * 8 + warp;
  if (row >= q1) return;
  const float* qr = p.q + (static_cast<size_t>(bh) * p.g.N_q + row) * D;
  const float* kb = p.k + static_cast<size_t>(bh) * p.g.N_k * D;
  const float* vb = p.v + static_cast<size_t>(bh) * p.g.N_k * D;
  const float* zp = p.z + bh * p.z_bh + t * p.z_t;
  const float* Sp = p.S + bh * p.S_bh + t * p.S_t;

  float qv[PER], acc[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    qv[i] = qr[lane + 32 * i];
    acc[i] = 0.f;
  }
  int any = 0;
  for (int e = lane; e < 2 * D; e += 32) any |= zp[e] > 0.f ? 1 : 0;
  const bool has_lin = __any_sync(kFull, any) != 0;

  const float scale = 1.0f / sqrtf(static_cast<float>(D));
  float m = has_lin ? 0.f : -INFINITY;
  float l = 0.f;
  for (int j = lo; j < hi; ++j) {
    const float* kr = kb + static_cast<size_t>(j) * D;
    float dot = 0.f;
#pragma unroll
    for (int i = 0; i < PER; ++i) dot += qv[i] * kr[lane + 32 * i];
    const float s = warp_sum(dot) * scale;
    if (s > m) {
      const float a = expf(m - s);
      l *= a;
#pragma unroll
      for (int i = 0; i < PER; ++i) acc[i] *= a;
      m = s;
    }
    const float w = expf(s - m);
    l += w;
    const float* vr = vb + static_cast<size_t>(j) * D;
#pragma unroll
    for (int i = 0; i < PER; ++i) acc[i] += w * vr[lane + 32 * i];
  }
  float num[PER], den = l;
#pragma unroll
  for (int i = 0; i < PER; ++i) num[i] = acc[i];
  if (has_lin) {
    float aL[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) aL[i] = 0.f;
    float nl = 0.f;
    const float* fq = p.phi_q ? p.phi_q + (static_cast<size_t>(bh) * p.g.N_q + row) * (2 * D) : nullptr;
#pragma unroll
    for (int idx = 0; idx < PER; ++idx) {
      for (int src = 0; src < 32; ++src) {
        const float x = __shfl_sync(kFull, qv[idx], src);
        const int dim = idx * 32 + src;
        float f1, f2;
        if (fq != nullptr) {  // precomputed (learned) features of q
          f1 = fq[dim];
          f2 = fq[D + dim];
        } else {
          f1 = psi_f32(x);
          f2 = f1 * f1;
        }
        nl += f1 * zp[dim] + f2 * zp[D + dim];
        const float* s1 = Sp + static_cast<size_t>(dim) * D;
        const float* s2 = Sp + static_cast<size_t>(D + dim) * D;
#pragma unroll
        for (int i = 0; i < PER; ++i) aL[i] += f1 * s1[lane + 32 * i] + f2 * s2[lane + 32 * i];
      }
    }
    const float sc = expf(-m);
#pragma unroll
    for (int i = 0; i < PER; ++i) num[i] += sc * aL[i];
    den += sc * nl;
  }
  float* orow = p.out + (static_cast<size_t>(bh) * p.g.N_q + row) * D;
#pragma unroll
  for (int i = 0; i < PER; ++i) orow[lane + 32 * i] = num[i] / den;
}

// One thread per state entry (e, c) of one segment (c == D: z), summing
// phi_e(k_j) v_jc over the segment's keys in order.
__global__ void __launch_bounds__(256) chunk_state_f32_kernel(const StateF32Params p) {
  const int D = p.D, W = D + 1;
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  const int s = blockIdx.y, bh = blockIdx.z;
  if (idx >= 2 * D * W) return;
  const int e = idx / W, c = idx % W;
  int a, b;
  p.sg.seg(s, a, b);
  const float* kb = p.k + static_cast<size_t>(bh) * p.sg.N_k * D;
  const float* vb = p.v + static_cast<size_t>(bh) * p.sg.N_k * D;
  const int dim = e < D ? e : e - D;
  float acc = 0.f;
  const float* fk = p.phi_k ? p.phi_k + static_cast<size_t>(bh) * p.sg.N_k * 2 * D : nullptr;
  for (int j = a; j < b; ++j) {
    float f;
    if (fk != nullptr) {  // precomputed (learned) features of k
      f = fk[static_cast<size_t>(j) * 2 * D + e];
    } else {
      f = psi_f32(kb[static_cast<size_t>(j) * D + dim]);
      if (e >= D) f = f * f;
    }
    acc += (c == D) ? f : f * vb[static_cast<size_t>(j) * D + c];
  }
  const size_t po = static_cast<size_t>(bh) * p.sg.n_seg + s;  // nsplit == 1
  if (c == D)
    p.part_z[po * 2 * D + e] = acc;
  else
    p.part_S[(po * 2 * D + e) * D + c] = acc;
}

// phi(x) = [psi(x), psi(x)^2] row-wise, x [rows, d] -> y [rows, 2d].
__global__ void phi_kernel(const void* x, int x_f32, void* y, int y_f32, long long rows, int d) {
  const long long n = rows * d;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long r = i / d;
    const int c = static_cast<int>(i % d);
    const float xv = x_f32 ? static_cast<const float*>(x)[i]
                           : __bfloat162float(static_cast<const __nv_bfloat16*>(x)[i]);
    const float f1 = psi_f32(xv), f2 = f1 * f1;
    const long long o1 = r * 2 * d + c, o2 = o1 + d;
    if (y_f32) {
      static_cast<float*>(y)[o1] = f1;
      static_cast<float*>(y)[o2] = f2;
    } else {
      static_cast<__nv_bfloat16*>(y)[o1] = __float2bfloat16_rn(f1);
      static_cast<__nv_bfloat16*>(y)[o2] = __float2bfloat16_rn(f2);
    }
  }
}

// Learned feature map (two-layer MLP, degree-2 features), fp32: a block
// takes MLP_ROWS rows; the hidden layer relu(W1 x + b1) goes through shared
// memory, then phi = [psi(u_1), psi(u_2)^2] of u = W2 h + b2.
constexpr int MLP_ROWS = 4;
__global__ void __launch_bounds__(256) phi_mlp_f32_kernel(const float* __restrict__ x, long long rows, int N, int H,
                                                          int d, const float* __restrict__ W1,
                                                          const float* __restrict__ b1,
                                                          const float* __restrict__ W2,
                                                          const float* __restrict__ b2, float* __restrict__ phi) {
  extern __shared__ float hid[];  // [MLP_ROWS][2d]
  const int d2 = 2 * d;
  const long long r0 = static_cast<long long>(blockIdx.x) * MLP_ROWS;
  for (int i = threadIdx.x; i < MLP_ROWS * d2; i += blockDim.x) {
    const int rr = i / d2, j = i % d2;
    const long long row = r0 + rr;
    float h = 0.f;
    if (row < rows) {
      const int head = static_cast<int>((row / N) % H);
      const float* w = W1 + (static_cast<size_t>(head) * d2 + j) * d;
      const float* xr = x + row * d;
      float a = b1[static_cast<size_t>(head) * d2 + j];
      for (int c = 0; c < d; ++c) a = fmaf(w[c], xr[c], a);
      h = fmaxf(a, 0.f);
    }
    hid[rr * d2 + j] = h;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < MLP_ROWS * d2; i += blockDim.x) {
    const int rr = i / d2, o = i % d2;
    const long long row = r0 + rr;
    if (row >= rows) continue;
    const int head = static_cast<int>((row / N) % H);
    const float* w = W2 + (static_cast<size_t>(head) * d2 + o) * d2;
    float u = b2[static_cast<size_t>(head) * d2 + o];
    for (int j = 0; j < d2; ++j) u = fmaf(w[j], hid[rr * d2 + j], u);
    const float f = psi_f32(u);
    phi[row * d2 + o] = (o < d) ? f : f * f;
  }
}

}  // namespace

cudaError_t launch_phi_mlp_f32(const float* x, long long rows, int N, int H, int d, const float* W1,
                               const float* b1, const float* W2, const float* b2, float* phi, cudaStream_t s) {
  const long long blocks = (rows + MLP_ROWS - 1) / MLP_ROWS;
  if (blocks <= 0) return cudaSuccess;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  phi_mlp_f32_kernel<<<static_cast<unsigned>(blocks), 256, MLP_ROWS * 2 * d * sizeof(float), s>>>(
      x, rows, N, H, d, W1, b1, W2, b2, phi);
  return cudaGetLastError();
}

cudaError_t launch_attention_f32(const AttnF32Params& p, int n_chunks, cudaStream_t s) {
  const int row_blocks = cdiv(p.g.step ? p.g.N_q : p.g.chunk_tok, 8);
  dim3 grid(row_blocks, n_chunks, p.BH);
  if (p.D == 128)
    attn_f32_kernel<4><<<grid, 256, 0, s>>>(p);
  else
    attn_f32_kernel<2><<<grid, 256, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_chunk_state_f32(const StateF32Params& p, cudaStream_t s) {
  if (p.sg.n_seg <= 0) return cudaSuccess;
  dim3 grid(cdiv(2 * p.D * (p.D + 1), 256), p.sg.n_seg, p.BH);
  chunk_state_f32_kernel<<<grid, 256, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_phi(const void* x, int x_f32, void* y, int y_f32, long long rows, int d, cudaStream_t s) {
  const long long n = rows * d;
  long long g = (n + 255) / 256;
  if (g > 148LL * 32) g = 148LL * 32;
  if (g < 1) g = 1;
  phi_kernel<<<static_cast<int>(g), 256, 0, s>>>(x, x_f32, y, y_f32, rows, d);
  return cudaGetLastError();
}

}  // namespace rehyat
