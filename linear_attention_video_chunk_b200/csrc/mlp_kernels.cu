// mlp_kernels.cu -- the learned feature map of "ReHyAt: Recurrent Hybrid
// Attention for Video Diffusion Transformers" (§4.3 Training specification,
// §7.1 Training Details: a two-layer MLP with degree-2 polynomial features,
// separate maps for queries and keys), i.e. the §3.2 feature-map equation
// with P = 2, on the tensor cores (tcgen05 / TMEM / TMA) for sm_100a.
#include <cstdint>

#include "geom.cuh"
#include "kernels.cuh"
#include "mlp.cuh"
#include "ptx.cuh"
#include "tc_common.cuh"

namespace rehyat {
namespace {

// 1 + elu of two values, the multiplies and adds done as packed fp32x2
// FMAs (x * log2e + 0 and x * 1 + 1 round exactly as the scalar multiply and
// add), squared as well for the psi^2 features.
__device__ __forceinline__ void psi_pair(float x0, float x1, bool square, float& f0, float& f1) {
  const uint64_t l2e2 = pack_f32x2(kLog2e, kLog2e), one2 = pack_f32x2(1.f, 1.f), zero2 = pack_f32x2(0.f, 0.f);
  float t0, t1, a0, a1;
  fma_f32x2(__float_as_uint(x0), __float_as_uint(x1), l2e2, zero2, t0, t1);
  fma_f32x2(__float_as_uint(x0), __float_as_uint(x1), one2, one2, a0, a1);
  f0 = x0 > 0.f ? a0 : ex2(t0);
  f1 = x1 > 0.f ? a1 : ex2(t1);
  if (square) fma_f32x2(__float_as_uint(f0), __float_as_uint(f1), pack_f32x2(f0, f1), zero2, f0, f1);
}

// ============================================================================
// Learned feature map: phi = [psi(u_1), psi(u_2)^2], u = W2 relu(W1 x + b1) + b2
// ============================================================================
// Two chained GEMMs per 128-row tile, both on the tensor cores with the
// head's weights resident in shared memory for the CTA's whole life:
//   H = x W1^T          (SS MMA, M = 128, N = 2D, K = D)    -> TMEM [0, 2D)
//   R = relu(H + b1)    bf16, written back into TMEM over H's columns
//   U = R W2^T          (TS MMA, M = 128, N = 2D, K = 2D)   -> TMEM [2D, 4D)
//   phi = [1 + elu(U_1 + b2_1), (1 + elu(U_2 + b2_2))^2]   bf16 -> global
// Warps 0-15 run both epilogues: warp w reads TMEM lane quarter w % 4 and
// column group w / 4 (a quarter of H's and of U's columns); warp 16 is the TMA
// producer, warp 17 the MMA issuer.  The next H GEMM (issued once the second
// GEMM, which reads R from H's columns, has completed) runs while the
// epilogue still reads U.  Features leave straight from registers: a thread
// holds 32 features (four 16-byte parts) of its row, the four threads of a
// lane quad exchange parts (a 4 x 4 transpose in two xor shuffles), and each
// store instruction then writes 64 contiguous bytes of each of 8 rows.  With
// no staging area in shared memory (at D = 128 the weights leave room for one
// x tile only) the next x tile loads as soon as the H GEMM has read the last.
template <int D>
struct MlpCfg {
  static constexpr int HID = 2 * D;                 // hidden width
  static constexpr int OUT = 2 * D;                 // feature width D'
  static constexpr int NBX = D / 64;                // 64-column boxes across x and W1
  static constexpr int NBH = HID / 64;              // ... across the hidden units (W2)
  static constexpr int XBOX = 128 * 128;            // 128 rows x 128 B
  static constexpr int X_BYTES = NBX * XBOX;
  static constexpr int W1BOX = HID * 128;           // HID rows x 128 B
  static constexpr int W2BOX = OUT * 128;
  static constexpr int W1_BYTES = NBX * W1BOX;
  static constexpr int W2_BYTES = NBH * W2BOX;
  static constexpr int NXB = (D == 128) ? 1 : 2;    // x tile buffers (the weights fill the rest)
  static constexpr int NG = 4;                      // epilogue column groups
  static constexpr int HG = HID / NG;               // hidden units of a group
  static constexpr int OG = OUT / NG;               // features of a group
  static constexpr int OFF_W1 = 0;
  static constexpr int OFF_W2 = W1_BYTES;
  static constexpr int OFF_X = OFF_W2 + W2_BYTES;
  static constexpr int OFF_BAR = OFF_X + NXB * X_BYTES;
  static constexpr int SMEM = OFF_BAR + 256 + 1024;
  static constexpr uint32_t TMEM_COLS = (HID + OUT <= 256) ? 256u : 512u;
  static constexpr int EPI_WARPS = 4 * NG;
  static constexpr int THREADS = 32 * EPI_WARPS + 64;
  // At D = 128 the second GEMM runs as two N = 128 halves of U (features
  // [0, D) and [D, 2D)), each with its own ready / free barrier, so the
  // features of the first half are computed while the tensor core produces
  // the second.  Epilogue group g takes features 32g.. of each half (one
  // 32-feature chunk a half).  At D = 64 a half would be 16 features a group,
  // under a chunk: one N = 2D GEMM, group g takes features g * OG...
  static constexpr bool SPLIT = (D == 128);
  static constexpr int NU = SPLIT ? 2 : 1;          // U halves
  static constexpr int B_W = 0, B_X = 1, B_XE = 1 + NXB, B_H = 1 + 2 * NXB, B_R = B_H + 1, B_U = B_H + 2,
                       B_UE = B_U + 2, B_FIN = B_UE + 2;
  static constexpr int NC = OG / 32;                // 32-feature chunk steps of a tile
  static_assert(!SPLIT || NC == NU, "one chunk per U half");
  static_assert(HG % 32 == 0 && OG % 32 == 0, "whole 32-column chunks per group");
  // both GEMMs: A and B K-major (x rows / R rows by W rows)
  static constexpr uint32_t IDESC1 = idesc_bf16_f32(128, HID, 0, 0);
  static constexpr uint32_t IDESC2 = idesc_bf16_f32(128, OUT / NU, 0, 0);
  static_assert(SMEM <= 232448, "shared memory");
  static_assert((B_FIN + 1) * 8 <= 128, "barrier area");
  static_assert(HID + OUT <= 512, "tensor memory");
};

template <int D>
__global__ void __launch_bounds__(MlpCfg<D>::THREADS, 1) phi_mlp_kernel(const __grid_constant__ MlpParams p) {
  using C = MlpCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int grp_id = blockIdx.x % p.groups;  // CTA = (map, bh, row group)
  const int rest = blockIdx.x / p.groups;
  const int bh = rest % p.BH;
  const int m = rest / p.BH;
  const int hh = bh % p.H, bb = bh / p.H;
  const int ntiles = cdiv(p.N, 128);
  const int my_tiles = grp_id < ntiles ? cdiv(ntiles - grp_id, p.groups) : 0;
  if (my_tiles == 0) return;  // uniform exit, before any barrier or TMEM use

  uint8_t* barea = smem + C::OFF_BAR;
  const uint32_t bar0 = smem_u32(barea);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(barea + 128);
  volatile int* abort = reinterpret_cast<volatile int*>(barea + 132);
#define BAR(i) (bar0 + 8u * static_cast<uint32_t>(i))
  if (threadIdx.x == 0) {
    mbar_init(BAR(C::B_W), 1);
    for (int i = 0; i < C::NXB; ++i) {
      mbar_init(BAR(C::B_X + i), 1);
      mbar_init(BAR(C::B_XE + i), 1);
    }
    mbar_init(BAR(C::B_H), 1);
    mbar_init(BAR(C::B_R), C::EPI_WARPS);
    for (int h = 0; h < 2; ++h) {
      mbar_init(BAR(C::B_U + h), 1);
      mbar_init(BAR(C::B_UE + h), C::EPI_WARPS);
    }
    mbar_init(BAR(C::B_FIN), 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == C::EPI_WARPS && lane == 0) {
    prefetch_tmap(&p.tm_x[m]);
    prefetch_tmap(&p.tm_w1[m]);
    prefetch_tmap(&p.tm_w2[m]);
  }
  if (warp == C::EPI_WARPS + 1) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < C::EPI_WARPS) {
    // ============================ epilogues ============================
    const int quarter = warp & 3, g = warp >> 2;
    const uint32_t lane_off = static_cast<uint32_t>(32 * quarter) << 16;
    const float4* b1 = reinterpret_cast<const float4*>(p.b1[m] + hh * C::HID + g * C::HG);  // group's hidden units
    const int odd = lane & 1, hi2 = (lane >> 1) & 1;  // position inside the lane quad
    // After a failed wait the remaining waits are skipped and the loop runs
    // out without blocking.
    bool ok = true;
    // phi = psi(U + b2), squared for the second half, one row a thread: the
    // 32 features of chunk c of tile t (for c = 0 and at D = 64 the group's
    // whole share; at D = 128 chunk c is read from U half c)
    auto feature_chunk = [&](int t, int c) {
      const int uh = C::SPLIT ? c : 0;  // U half of this chunk
      const int fc = C::SPLIT ? c * (C::OUT / 2) + 32 * g : g * C::OG + 32 * c;  // its first feature
      if (C::SPLIT || c == 0) {
        ok = ok && warp_wait(BAR(C::B_U + uh), t & 1, abort);
        if (c == 0 && threadIdx.x == 0) TRACE(2, t);
        tc_fence_after();
      }
      uint32_t v[32];
      tmem_ld32(tmem + lane_off + C::HID + fc, v);
      tmem_ld_wait();
      reg_fence(v);
      if (C::SPLIT || c == C::NC - 1) {  // U (half) fully read: the next tile's GEMM may overwrite it
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(C::B_UE + uh));
      }
      const float4* b2 = reinterpret_cast<const float4*>(p.b2[m] + hh * C::OUT + fc);
      const bool square = fc >= D;  // features D..2D-1 are psi_2^2
      uint32_t o[16];
#pragma unroll
      for (int q4 = 0; q4 < 8; ++q4) {
        const float4 bv = __ldg(b2 + q4);
        const uint64_t one2 = pack_f32x2(1.f, 1.f);
        float u0, u1, u2, u3;  // U + b2
        fma_f32x2(v[4 * q4], v[4 * q4 + 1], one2, pack_f32x2(bv.x, bv.y), u0, u1);
        fma_f32x2(v[4 * q4 + 2], v[4 * q4 + 3], one2, pack_f32x2(bv.z, bv.w), u2, u3);
        float f0, f1, f2, f3;
        psi_pair(u0, u1, square, f0, f1);
        psi_pair(u2, u3, square, f2, f3);
        o[2 * q4] = pack_bf16(f0, f1);
        o[2 * q4 + 1] = pack_bf16(f2, f3);
      }
      if (c == 0 && threadIdx.x == 0) TRACE(3, t);
      // 4 x 4 transpose of 16-byte parts inside the lane quad: lane 4q + i
      // then holds part i (features 8i..8i+7) of rows 4q..4q+3 of the warp's
      // 32, part k of row 4q + k in P[k]
      uint4 P[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) P[j] = make_uint4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
      {
        const uint4 r0 = shfl_xor_u4(odd ? P[0] : P[1], 1), r1 = shfl_xor_u4(odd ? P[2] : P[3], 1);
        if (odd) {
          P[0] = r0;
          P[2] = r1;
        } else {
          P[1] = r0;
          P[3] = r1;
        }
      }
      {
        const uint4 r0 = shfl_xor_u4(hi2 ? P[0] : P[2], 2), r1 = shfl_xor_u4(hi2 ? P[1] : P[3], 2);
        if (hi2) {
          P[0] = r0;
          P[1] = r1;
        } else {
          P[2] = r0;
          P[3] = r1;
        }
      }
      const int row0 = 128 * (grp_id + t * p.groups) + 32 * quarter + 4 * (lane >> 2);
      __nv_bfloat16* dst = p.phi[m] + (static_cast<size_t>(bh) * p.N + row0) * C::OUT + fc + 8 * (lane & 3);
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (row0 + k < p.N) *reinterpret_cast<uint4*>(dst + static_cast<size_t>(k) * C::OUT) = P[k];
      if (c == 0 && threadIdx.x == 0) TRACE(4, t);
    };
    // Per tile: R, then (at D = 128) the previous tile's second chunk, during
    // which the tensor core computes this tile's first U half, then this
    // tile's first chunk, during which it computes the second U half and the
    // next tile's H.
    for (int it = 0; it < my_tiles; ++it) {
      ok = ok && warp_wait(BAR(C::B_H), it & 1, abort);
      if (threadIdx.x == 0) TRACE(0, it);
      tc_fence_after();
      // R = relu(H + b1) as bf16 pairs: the group's HG hidden units go to the
      // first HG/2 of its own HG columns (chunk c is read before any column it
      // overwrites, and the groups' column ranges are disjoint)
#pragma unroll 1
      for (int c = 0; c < C::HG / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_off + g * C::HG + 32 * c, v);
        tmem_ld_wait();
        reg_fence(v);
        uint32_t rr[16];
#pragma unroll
        for (int q4 = 0; q4 < 8; ++q4) {
          const float4 bv = __ldg(b1 + 8 * c + q4);
          const uint64_t one2 = pack_f32x2(1.f, 1.f);
          float h0, h1, h2, h3;  // H + b1 (x * 1 + b rounds as x + b)
          fma_f32x2(v[4 * q4], v[4 * q4 + 1], one2, pack_f32x2(bv.x, bv.y), h0, h1);
          fma_f32x2(v[4 * q4 + 2], v[4 * q4 + 3], one2, pack_f32x2(bv.z, bv.w), h2, h3);
          rr[2 * q4] = pack_bf16(fmaxf(h0, 0.f), fmaxf(h1, 0.f));
          rr[2 * q4 + 1] = pack_bf16(fmaxf(h2, 0.f), fmaxf(h3, 0.f));
        }
        tmem_st16(tmem + lane_off + g * C::HG + 16 * c, rr);
      }
      warp_release(BAR(C::B_R), lane);
      if (threadIdx.x == 0) TRACE(1, it);
      if (C::SPLIT) {
        if (it > 0) feature_chunk(it - 1, 1);
        feature_chunk(it, 0);
      } else {
#pragma unroll 1
        for (int c = 0; c < C::NC; ++c) feature_chunk(it, c);
      }
    }
    if (C::SPLIT) feature_chunk(my_tiles - 1, 1);
  } else if (warp == C::EPI_WARPS) {
    // ========================= TMA producer: x tiles =========================
    if (lane == 0) {
      mbar_arrive_expect_tx(BAR(C::B_W), C::W1_BYTES + C::W2_BYTES);
      for (int b = 0; b < C::NBX; ++b)
        tma_load_3d(smem_u32(smem + C::OFF_W1 + b * C::W1BOX), &p.tm_w1[m], BAR(C::B_W), 64 * b, 0, hh);
      for (int b = 0; b < C::NBH; ++b)
        tma_load_3d(smem_u32(smem + C::OFF_W2 + b * C::W2BOX), &p.tm_w2[m], BAR(C::B_W), 64 * b, 0, hh);
      bool ok = true;
      int loaded = 0;  // x tiles issued
      // x tile `it` into its slot once the H GEMM of the slot's previous tile
      // has read it
      for (int it = 0; it < my_tiles && ok; ++it) {
        const int slot = it % C::NXB;
        ok = mbar_wait(BAR(C::B_XE + slot), ((it / C::NXB) & 1) ^ 1, abort);
        if (!ok) break;
        TRACE(11, it);
        const uint32_t dst = smem_u32(smem + C::OFF_X + slot * C::X_BYTES);
        mbar_arrive_expect_tx(BAR(C::B_X + slot), C::X_BYTES);
        for (int b = 0; b < C::NBX; ++b)
          tma_load_4d(dst + b * C::XBOX, &p.tm_x[m], BAR(C::B_X + slot), 64 * b, 128 * (grp_id + it * p.groups), hh,
                      bb);
        loaded = it + 1;
      }
      drain_wait(BAR(C::B_W), 0);
      for (int i2 = (loaded > C::NXB ? loaded - C::NXB : 0); i2 < loaded; ++i2)
        drain_wait(BAR(C::B_X + i2 % C::NXB), (i2 / C::NXB) & 1);
    }
  } else {
    // ============================ MMA issuer ============================
    if (lane == 0) {
      constexpr uint32_t HI = desc_hi_sw128(1024);  // K-major: 8-row groups 1024 B apart
      const uint32_t lo_w1 = desc_lo(smem_u32(smem + C::OFF_W1), 16);
      const uint32_t lo_w2 = desc_lo(smem_u32(smem + C::OFF_W2), 16);
      bool ok = mbar_wait(BAR(C::B_W), 0, abort);
      for (int it = 0; it < my_tiles && ok; ++it) {
        const int slot = it % C::NXB;
        ok = mbar_wait(BAR(C::B_X + slot), (it / C::NXB) & 1, abort);
        // H overwrites the TMEM columns that hold R of the previous tile, the
        // A operand of its second GEMM: issued only once that GEMM has
        // completed (tcgen05 operands must not change under an MMA in flight)
        if (ok && it > 0) ok = mbar_wait(BAR(C::B_U + C::NU - 1), (it - 1) & 1, abort);
        if (!ok) break;
        TRACE(8, it);
        tc_fence_after();
        const uint32_t lo_x = desc_lo(smem_u32(smem + C::OFF_X + slot * C::X_BYTES), 16);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)  // K-step kk: box kk/4, 32 B into the swizzled row
          mma_ss(tmem, desc_join(lo_x + (((kk >> 2) * C::XBOX + (kk & 3) * 32) >> 4), HI),
                 desc_join(lo_w1 + (((kk >> 2) * C::W1BOX + (kk & 3) * 32) >> 4), HI), C::IDESC1, kk > 0 ? 1u : 0u);
        mma_commit(BAR(C::B_XE + slot));
        mma_commit(BAR(C::B_H));
        TRACE(9, it);
        // R of this tile written; each U half once the previous tile's
        // features of that half have been read out of it
        ok = mbar_wait(BAR(C::B_R), it & 1, abort);
        for (int h = 0; h < C::NU && ok; ++h) {
          ok = mbar_wait(BAR(C::B_UE + h), (it & 1) ^ 1, abort);
          if (!ok) break;
          if (h == 0) TRACE(10, it);
          tc_fence_after();
          const uint32_t wrow = (h * (C::OUT / C::NU) * 128) >> 4;  // the half's first W2 row
#pragma unroll
          for (int kk = 0; kk < C::HID / 16; ++kk) {  // 16 hidden units = 8 packed columns of R
            const uint32_t a = tmem + (kk / (C::HG / 16)) * C::HG + (kk % (C::HG / 16)) * 8;
            mma_ts(tmem + C::HID + h * (C::OUT / C::NU), a,
                   desc_join(lo_w2 + wrow + (((kk >> 2) * C::W2BOX + (kk & 3) * 32) >> 4), HI), C::IDESC2,
                   kk > 0 ? 1u : 0u);
          }
          mma_commit(BAR(C::B_U + h));
        }
      }
      mma_commit(BAR(C::B_FIN));
      drain_wait(BAR(C::B_FIN), 0);
    }
  }
#undef BAR
  tc_fence_before();
  __syncthreads();
  if (warp == C::EPI_WARPS + 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace

template <int D>
static cudaError_t launch_mlp_t(const MlpParams& p, int n_maps, cudaStream_t s) {
  auto* k = phi_mlp_kernel<D>;
  cudaError_t e = prepare_kernel_once(reinterpret_cast<const void*>(k), MlpCfg<D>::SMEM, 0);
  if (e != cudaSuccess) return e;
  k<<<n_maps * p.BH * p.groups, MlpCfg<D>::THREADS, MlpCfg<D>::SMEM, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_phi_mlp(int D, const MlpParams& p, int n_maps, cudaStream_t s) {
  if (p.N <= 0 || n_maps <= 0) return cudaSuccess;
  return D == 128 ? launch_mlp_t<128>(p, n_maps, s) : launch_mlp_t<64>(p, n_maps, s);
}

cudaError_t read_and_clear_device_error_mlp(unsigned int* v) {
  cudaError_t e = cudaMemcpyFromSymbol(v, g_device_error, sizeof(unsigned int));
  if (e != cudaSuccess) return e;
  const unsigned int zero = 0;
  return cudaMemcpyToSymbol(g_device_error, &zero, sizeof(unsigned int));
}

}  // namespace rehyat
