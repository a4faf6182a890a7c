// tc_kernels.cu -- tensor-core (tcgen05 / TMEM / TMA) kernels for sm_100a.
//
// 1. hybrid_chunk_attn_kernel: the fused per-chunk hybrid attention of
//    "ReHyAt: Recurrent Hybrid Attention for Video Diffusion Transformers",
//    §3.2 (joint normaliser y = (a^S + a^L) / (n^S + n^L)) over the §3.3
//    sets: exact softmax over the chunk's window [lo_t, hi_t) plus the linear
//    term phi(q) S_t, phi(q) z_t of every earlier key (§3.1 caching).
// (The segment states that feed the linear term are computed in
// state_tc_kernels.cu.)
//
// Layout conventions (all operand tiles use the 128-byte TMA swizzle):
//   a "box" is 128 B wide (64 bf16) and R rows tall; row r lives at r*128 and
//   its 16-byte chunk c at ((c ^ (r & 7)) * 16).  A D-wide tile is D/64 boxes.
#include <cstdint>

#include "kernels.cuh"
#include "ptx.cuh"
#include "tc_common.cuh"

namespace rehyat {
namespace {

// P = 2^(s * scale - m) for one half (64 keys) of a 128-key row tile, packed
// to bf16 pairs and stored into TMEM columns [32*HALF, 32*HALF + 32) of S;
// returns the row sum of exactly the stored bf16 values.
template <int HALF>
__device__ __forceinline__ float exp_pack_store(uint32_t (&s)[4][32], float scale, float neg_m, uint32_t tS) {
  float rsum[4] = {0.f, 0.f, 0.f, 0.f};  // independent partial sums
  uint32_t pk[32];
  const uint64_t sc2 = pack_f32x2(scale, scale), nm2 = pack_f32x2(neg_m, neg_m);
#pragma unroll
  for (int a = 2 * HALF; a < 2 * HALF + 2; ++a) {
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      // x = s * scale - m for two keys in one packed fp32x2 FMA (measured
      // 2% faster for the whole kernel than two scalar FMAs)
      float x0, x1;
      fma_f32x2(s[a][2 * c], s[a][2 * c + 1], sc2, nm2, x0, x1);
      const float p0 = ex2(x0);
      const float p1 = ex2(x1);
      const uint32_t u = pack_bf16(p0, p1);
      // the denominator sums exactly the bf16 weights the P.V MMA uses
      float& acc = rsum[c & 3];
      acc = add_bf16_hi(u, add_bf16_lo(u, acc));
      pk[(a & 1) * 16 + c] = u;
    }
  }
  tmem_st32(tS + 32 * HALF, pk);
  return (rsum[0] + rsum[1]) + (rsum[2] + rsum[3]);
}


// ============================================================================
// Fused chunk attention
// ============================================================================
template <int D>
struct AttnCfg {
  static constexpr int NBOX = D / 64;
  static constexpr int BOX_BYTES = 128 * 128;               // 128 rows x 128 B
  static constexpr int TILE_BYTES = NBOX * BOX_BYTES;       // 128 x D bf16
  static constexpr int NSLOTS = (D == 128) ? 5 : 8;         // K/V/state ring
  static constexpr int SPP = (2 * D) / 128;                 // state slots per hi|lo part
  static constexpr int OFF_RING = 0;                        // ring first, then the Q tiles:
  static constexpr int OFF_Q = NSLOTS * TILE_BYTES;         // operand reads stay inside the
  static constexpr int OFF_BAR = OFF_Q + 2 * TILE_BYTES;    // data area whatever the layout
  static constexpr int SMEM = OFF_BAR + 512 + 1024;         // + barriers, + alignment slack
  // barrier indices
  static constexpr int B_Q = 0;
  static constexpr int B_FULL = 1;
  static constexpr int B_EMPTY = B_FULL + NSLOTS;
  static constexpr int B_S = B_EMPTY + NSLOTS;   // [2] scores ready in TMEM
  static constexpr int B_P = B_S + 2;            // [2] first 64 keys of P written to TMEM
  static constexpr int B_P1 = B_P + 2;           // [2] last 64 keys of P written to TMEM
  static constexpr int B_O = B_P1 + 2;           // [2] last P.V done
  static constexpr int B_PHI = B_O + 2;          // [2] scaled phi(Q) written to TMEM
  static constexpr int B_LIN = B_PHI + 2;        // [2] linear MMA done
  static constexpr int B_PVD = B_LIN + 2;        // [2] P.V of the current key tile done
  static constexpr int B_FIN = B_PVD + 2;        // MMA drain
  static constexpr int NBARS = B_FIN + 1;
  static_assert(NBARS * 8 <= 256, "barrier area");
  static_assert(SMEM <= 232448, "shared memory");
  // TMEM columns: S/P of tile X at X*128, O of tile X at 256 + X*D.
  static constexpr uint32_t TMEM_COLS = 512;
  // 12 warps: warpgroups 0 and 1 run the softmax of query tiles A and B,
  // warpgroup 2 holds the TMA producer (warp 8) and the MMA issuer (warp 9).
  // Launched at 168 registers a thread (65536 / 384, rounded down to 8);
  // warpgroup 2 gives registers to the softmax warpgroups:
  // 2 * 128 * REGS_SOFTMAX + 128 * REGS_ISSUE == 384 * REGS_LAUNCH.
  static constexpr int THREADS = 384;
  static constexpr uint32_t REGS_LAUNCH = 168;
  static constexpr uint32_t REGS_SOFTMAX = 176;
  static constexpr uint32_t REGS_ISSUE = 152;
  static_assert(2 * 128 * REGS_SOFTMAX + 128 * REGS_ISSUE == THREADS * REGS_LAUNCH, "register split");
  static constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 128, 0, 0);  // Q K^T: both K-major
  static constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, D, 0, 1);   // P V, phi~ S: B MN-major
};

// events: softmax of tile X (lane 0 of warp 4X): 0+5X S ready seen, 1+5X S in
// registers, 2+5X max done, 3+5X first P half released, 4+5X P released; MMA issuer:
// 10+X P_X seen, 12+X S_X(j+1) issued, 14 unit start (j = 0), Q and K_0 in
// (j = 1), K_{j+1} in (j + 2), 15 P_A.V_j issued

// PHI: the linear term takes phi(q) rows precomputed by a learned feature map
// (p.phi_q) instead of evaluating the fixed phi on the Q tile.
template <int D, bool PARTS, bool PHI>
__global__ void __launch_bounds__(384, 1) hybrid_chunk_attn_kernel(const __grid_constant__ AttnParams p) {
  using C = AttnCfg<D>;
  constexpr int NS = C::NSLOTS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // A kernel launched behind this one with a programmatic dependency (the
  // recurrent step's fold of evicted keys) may be scheduled once every CTA
  // has started: it reads nothing this kernel writes.
  grid_dep_launch();

  // ---- unit -> (bh, chunk t, pair of 128-row query tiles) -----------------
  // Chunks are visited 1, 2, ..., n-1, 0: chunk 0 has no overlap frames (the
  // shortest window), so the longest units start first.  A split unit's two
  // CTAs (half 0 and 1) each take half of the key window's tiles.
  const int u = blockIdx.x;
  int ou = u, half = -1;
  if (p.n_split > 0 && u >= p.split_begin) {
    const int v = u - p.split_begin;
    if (v < 2 * p.n_split) {
      ou = p.split_begin + (v >> 1);
      half = v & 1;
    } else {
      ou = u - p.n_split;
    }
  }
  int pair, bh, t;
  if (p.pair_major) {
    pair = ou / p.BH;
    bh = ou % p.BH;
    t = 0;
  } else {
    pair = ou % p.pairs;
    const int rest = ou / p.pairs;
    bh = rest % p.BH;
    const int o = rest / p.BH;
    t = (p.g.n_chunks > 1) ? (o + 1) % p.g.n_chunks : 0;
  }
  int q0, q1, lo, hi;
  p.g.chunk(t, q0, q1, lo, hi);
  if (half >= 0) {
    const int h0 = (cdiv(hi - lo, 128) + 1) / 2;  // tiles of the first half
    if (half == 0)
      hi = lo + 128 * h0;
    else
      lo += 128 * h0;
  }
  const int rowA0 = q0 + pair * 256;
  const int rowB0 = rowA0 + 128;
  const int nA = imin(imax(q1 - rowA0, 0), 128);
  const int nB = imin(imax(q1 - rowB0, 0), 128);
  if (nA <= 0) return;  // the ragged last chunk has fewer tiles (uniform exit)
  const bool hasB = nB > 0;
  const int win = hi - lo;  // >= 1
  const int ntiles = cdiv(win, 128);

  uint8_t* barea = smem + C::OFF_BAR;
  const uint32_t bar0 = smem_u32(barea);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(barea + 256);
  volatile int* abort = reinterpret_cast<volatile int*>(barea + 260);
  int* lin_flag = reinterpret_cast<int*>(barea + 264);
#define BAR(i) (bar0 + 8u * static_cast<uint32_t>(i))

  if (threadIdx.x == 0) {
    mbar_init(BAR(C::B_Q), 1);
    for (int i = 0; i < NS; ++i) {
      mbar_init(BAR(C::B_FULL + i), 1);
      mbar_init(BAR(C::B_EMPTY + i), 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(BAR(C::B_S + x), 1);
      mbar_init(BAR(C::B_P + x), 4);           // one arrive per softmax warp
      mbar_init(BAR(C::B_P1 + x), 4);
      mbar_init(BAR(C::B_O + x), 1);
      mbar_init(BAR(C::B_PHI + x), 4);
      mbar_init(BAR(C::B_LIN + x), 1);
      mbar_init(BAR(C::B_PVD + x), 1);
    }
    mbar_init(BAR(C::B_FIN), 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    // The linear set is non-empty iff z_t > 0 somewhere (phi > 0 elementwise).
    int f = 0;
    if (p.z != nullptr && half != 1) {  // the linear term is added by the first half of a split unit
      const float* zp = p.z + bh * p.z_bh + t * p.z_t;
      for (int e = lane; e < 2 * D; e += 32) f |= (zp[e] > 0.f) ? 1 : 0;
    }
    f = __any_sync(kFull, f);
    if (lane == 0) *lin_flag = f;
  }
  if (warp == 8 && lane == 0) {
    prefetch_tmap(&p.tm_q);
    prefetch_tmap(&p.tm_k);
    prefetch_tmap(&p.tm_v);
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const bool has_lin = (*lin_flag) != 0;
  if (warp < 8)
    regs_increase<C::REGS_SOFTMAX>();
  else
    regs_decrease<C::REGS_ISSUE>();

  if (warp < 8) {
    // ======================= softmax / epilogue warps =======================
    const int X = warp >> 2;  // query tile A (0) or B (1)
    const int wl = warp & 3;  // TMEM lane quarter
    const int nX = X ? nB : nA;
    if (X == 0 || hasB) {
      const int r = wl * 32 + lane;  // row inside the 128-row tile
      const uint32_t lane_off = static_cast<uint32_t>(wl * 32) << 16;
      const uint32_t tS = tmem + lane_off + X * 128;
      const uint32_t tO = tmem + lane_off + 256 + X * D;
      // Running shift (log2 units).  With a non-empty linear set it starts
      // at 0, so the final shift M = max(m, 0) keeps exp(-M) <= 1 on the
      // linear terms; without one it is the usual running maximum.
      float m_used = has_lin ? 0.f : -INFINITY;
      float l = 0.f;
      bool ok = true;
      for (int j = 0; j < ntiles; ++j) {
        ok = warp_wait(BAR(C::B_S + X), j & 1, abort);
        if (!ok) break;
        if (wl == 0 && lane == 0) TRACE(0 + 5 * X, j);
        tc_fence_after();
        uint32_t s[4][32];
        tmem_ld32(tS + 0, s[0]);
        tmem_ld32(tS + 32, s[1]);
        tmem_ld32(tS + 64, s[2]);
        tmem_ld32(tS + 96, s[3]);
        tmem_ld_wait();
        reg_fence(s[0]);
        reg_fence(s[1]);
        reg_fence(s[2]);
        reg_fence(s[3]);
        if (wl == 0 && lane == 0) TRACE(1 + 5 * X, j);
        const int valid = win - j * 128;  // keys of this tile inside the window
        if (valid < 128) {                 // only the window's last tile is partial
#pragma unroll
          for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int c = 0; c < 32; ++c)
              if (a * 32 + c >= valid) s[a][c] = __float_as_uint(-INFINITY);
        }
        // Row max on raw scores (scale > 0): eight independent chains of
        // three-input max, then a short tree.
        float mr[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int a = i >> 1, c0 = (i & 1) * 16;
          float m = fmax3(__uint_as_float(s[a][c0]), __uint_as_float(s[a][c0 + 1]), __uint_as_float(s[a][c0 + 2]));
#pragma unroll
          for (int c = 3; c < 15; c += 2)
            m = fmax3(m, __uint_as_float(s[a][c0 + c]), __uint_as_float(s[a][c0 + c + 1]));
          mr[i] = fmaxf(m, __uint_as_float(s[a][c0 + 15]));
        }
        const float mraw = fmaxf(fmax3(fmax3(mr[0], mr[1], mr[2]), fmax3(mr[3], mr[4], mr[5]), mr[6]), mr[7]);
        const float mx = mraw * p.scale_log2;
        if (wl == 0 && lane == 0) TRACE(2 + 5 * X, j);
        // Lazy rescaling: move the shift only when the row maximum exceeds
        // it by more than 2^8, so P <= 256 and fp32 sums stay exact enough.
        const bool need = mx > m_used + 8.f;
        const bool warp_need = __any_sync(kFull, need) != 0;
        const float mnew = need ? mx : m_used;
        const float alpha = need ? ex2(m_used - mnew) : 1.f;
        m_used = mnew;
        const float neg_m = -m_used;
        // P is released in two 64-key halves, so the first half's P.V runs
        // on the tensor core while the second half's exponentials are taken
        // (masked keys of the window's partial last tile give 0).
        float rs = exp_pack_store<0>(s, p.scale_log2, neg_m, tS);
        if (warp_need && j > 0) {
          // O holds tiles 0..j-1 (their P.V completed before S_j was
          // signalled) and must move to the new shift before P_j.V_j.
          // (Done after the first half's exponentials, whose scores no
          // longer occupy registers.)
#pragma unroll
          for (int a = 0; a < D / 32; ++a) {
            uint32_t ov[32];
            tmem_ld32(tO + 32 * a, ov);
            tmem_ld_wait();
            reg_fence(ov);
#pragma unroll
            for (int c = 0; c < 32; ++c) ov[c] = __float_as_uint(__uint_as_float(ov[c]) * alpha);
            tmem_st32(tO + 32 * a, ov);
          }
        }
        warp_release(BAR(C::B_P + X), lane);
        if (wl == 0 && lane == 0) TRACE(3 + 5 * X, j);
        rs += exp_pack_store<1>(s, p.scale_log2, neg_m, tS);
        warp_release(BAR(C::B_P1 + X), lane);
        if (wl == 0 && lane == 0) TRACE(4 + 5 * X, j);
        l = l * alpha + rs;
      }

      if (ok) ok = warp_wait(BAR(C::B_O + X), 0, abort);
      tc_fence_after();
      const bool vrow = r < nX;
      const int qrow = (X ? rowB0 : rowA0) + r;
      const size_t grow = static_cast<size_t>(bh) * p.g.N_q + qrow;  // [BH, N_q] index (parts)

      if (PARTS && ok) {
#pragma unroll
        for (int a = 0; a < D / 32; ++a) {
          uint32_t ov[32];
          tmem_ld32(tO + 32 * a, ov);
          tmem_ld_wait();
          reg_fence(ov);
          if (vrow) {
            float4* dst = reinterpret_cast<float4*>(p.aS + grow * D + 32 * a);
#pragma unroll
            for (int c = 0; c < 8; ++c)
              dst[c] = make_float4(__uint_as_float(ov[4 * c]), __uint_as_float(ov[4 * c + 1]),
                                   __uint_as_float(ov[4 * c + 2]), __uint_as_float(ov[4 * c + 3]));
          }
        }
        if (vrow) {
          p.nS[grow] = l;
          p.Mo[grow] = m_used * kLn2;
        }
      }

      // ---- linear term: phi(q) S_t and phi(q) z_t (§3.1 cached sums) ----
      float nl = 0.f;  // e^{-M} phi(q) z_t
      if (has_lin && ok) {
        const float sc = ex2(-m_used);  // exp(-M), <= 1
        const float* zp = p.z + bh * p.z_bh + t * p.z_t;
        if constexpr (PHI) {
          // phi(q) row of 2D bf16 features: [0, D) into columns [0, D/2),
          // [D, 2D) into [D/2, D), two features a column
          const uint4* fr = reinterpret_cast<const uint4*>(p.phi_q) +
                            (static_cast<size_t>(bh) * p.g.N_q + (vrow ? qrow : 0)) * (2 * D / 8);
#pragma unroll
          for (int b = 0; b < C::NBOX; ++b) {
            uint32_t pa[32], pb[32];
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) {
              const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);
              const uint4 ra = vrow ? __ldg(fr + 8 * b + cc) : z4;
              const uint4 rb = vrow ? __ldg(fr + D / 8 + 8 * b + cc) : z4;
              const uint32_t wa[4] = {ra.x, ra.y, ra.z, ra.w};
              const uint32_t wb[4] = {rb.x, rb.y, rb.z, rb.w};
#pragma unroll
              for (int h = 0; h < 4; ++h) {
                const int dim = 64 * b + 8 * cc + 2 * h;
                const uint32_t ua = pack_bf16(bf16lo(wa[h]) * sc, bf16hi(wa[h]) * sc);
                const uint32_t ub = pack_bf16(bf16lo(wb[h]) * sc, bf16hi(wb[h]) * sc);
                nl += bf16lo(ua) * zp[dim] + bf16hi(ua) * zp[dim + 1] + bf16lo(ub) * zp[D + dim] +
                      bf16hi(ub) * zp[D + dim + 1];
                pa[cc * 4 + h] = ua;
                pb[cc * 4 + h] = ub;
              }
            }
            tmem_st32(tS + 32 * b, pa);
            tmem_st32(tS + D / 2 + 32 * b, pb);
          }
        } else {
        const uint8_t* qrow = smem + C::OFF_Q + X * C::TILE_BYTES + r * 128;
#pragma unroll
        for (int b = 0; b < C::NBOX; ++b) {
          uint32_t pa[32], pb[32];
#pragma unroll
          for (int cc = 0; cc < 8; ++cc) {
            const uint4 raw =
                *reinterpret_cast<const uint4*>(qrow + b * C::BOX_BYTES + ((cc ^ (r & 7)) << 4));
            const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              const float s0 = psi1(bf16lo(w[h]));
              const float s1 = psi1(bf16hi(w[h]));
              const int dim = 64 * b + 8 * cc + 2 * h;
              const uint32_t ua = pack_bf16(s0 * sc, s1 * sc);
              const uint32_t ub = pack_bf16((s0 * s0) * sc, (s1 * s1) * sc);
              // n^L e^{-M} from the same bf16 features the phi~ S MMA uses
              nl += bf16lo(ua) * zp[dim] + bf16hi(ua) * zp[dim + 1] + bf16lo(ub) * zp[D + dim] +
                    bf16hi(ub) * zp[D + dim + 1];
              pa[cc * 4 + h] = ua;
              pb[cc * 4 + h] = ub;
            }
          }
          // features psi (0..D-1) then psi^2 (D..2D-1), two per column
          tmem_st32(tS + 32 * b, pa);
          tmem_st32(tS + D / 2 + 32 * b, pb);
        }
        }
        warp_release(BAR(C::B_PHI + X), lane);
        ok = warp_wait(BAR(C::B_LIN + X), 0, abort);
        tc_fence_after();
      }

      if (ok && !PARTS && half >= 0) {
        // split unit: the partial row (unnormalised O, its denominator and
        // shift, log2 units) for the merge
        float* e = p.part + ((static_cast<size_t>((ou - p.split_begin) * 2 + half) * 2 + X) * 128 + r) * (D + 4);
#pragma unroll
        for (int a = 0; a < D / 32; ++a) {
          uint32_t ov[32];
          tmem_ld32(tO + 32 * a, ov);
          tmem_ld_wait();
          reg_fence(ov);
          float4* dst = reinterpret_cast<float4*>(e + 32 * a);
#pragma unroll
          for (int c = 0; c < 8; ++c)
            dst[c] = make_float4(__uint_as_float(ov[4 * c]), __uint_as_float(ov[4 * c + 1]),
                                 __uint_as_float(ov[4 * c + 2]), __uint_as_float(ov[4 * c + 3]));
        }
        e[D] = l + nl;
        e[D + 1] = m_used;
      } else if (ok) {
        if (!PARTS) {
          const float inv = 1.f / (l + nl);
#pragma unroll
          for (int a = 0; a < D / 32; ++a) {
            uint32_t ov[32];
            tmem_ld32(tO + 32 * a, ov);
            tmem_ld_wait();
            reg_fence(ov);
            if (vrow) {
              uint4* dst = reinterpret_cast<uint4*>(p.out + (bh / p.H) * p.o_sb + (bh % p.H) * p.o_sh +
                                                    qrow * p.o_sr + 32 * a);
#pragma unroll
              for (int c = 0; c < 4; ++c) {
                uint4 w;
                w.x = pack_bf16(__uint_as_float(ov[8 * c + 0]) * inv, __uint_as_float(ov[8 * c + 1]) * inv);
                w.y = pack_bf16(__uint_as_float(ov[8 * c + 2]) * inv, __uint_as_float(ov[8 * c + 3]) * inv);
                w.z = pack_bf16(__uint_as_float(ov[8 * c + 4]) * inv, __uint_as_float(ov[8 * c + 5]) * inv);
                w.w = pack_bf16(__uint_as_float(ov[8 * c + 6]) * inv, __uint_as_float(ov[8 * c + 7]) * inv);
                dst[c] = w;
              }
            }
          }
        } else {
#pragma unroll
          for (int a = 0; a < D / 32; ++a) {
            uint32_t ov[32];
            if (has_lin) {
              tmem_ld32(tO + 32 * a, ov);
              tmem_ld_wait();
              reg_fence(ov);
            } else {
#pragma unroll
              for (int c = 0; c < 32; ++c) ov[c] = 0u;
            }
            if (vrow) {
              float4* dst = reinterpret_cast<float4*>(p.aL + grow * D + 32 * a);
#pragma unroll
              for (int c = 0; c < 8; ++c)
                dst[c] = make_float4(__uint_as_float(ov[4 * c]), __uint_as_float(ov[4 * c + 1]),
                                     __uint_as_float(ov[4 * c + 2]), __uint_as_float(ov[4 * c + 3]));
            }
          }
          if (vrow) p.nL[grow] = nl;
        }
      }
    }
  } else if (warp == 8) {
    // =============================== TMA producer ============================
    if (lane == 0) {
      const uint32_t sq = smem_u32(smem + C::OFF_Q);
      const uint32_t ring = smem_u32(smem + C::OFF_RING);
      const int hh = bh % p.H, bb = bh / p.H;
      mbar_arrive_expect_tx(BAR(C::B_Q), (hasB ? 2 : 1) * C::TILE_BYTES);
      for (int b = 0; b < C::NBOX; ++b) tma_load_4d(sq + b * C::BOX_BYTES, &p.tm_q, BAR(C::B_Q), 64 * b, rowA0, hh, bb);
      if (hasB)
        for (int b = 0; b < C::NBOX; ++b)
          tma_load_4d(sq + C::TILE_BYTES + b * C::BOX_BYTES, &p.tm_q, BAR(C::B_Q), 64 * b, rowB0, hh, bb);
      uint32_t seq = 0;
      bool ok = true;
      // zc >= 0: a state tile (3-D map, depth zc); else a K/V tile (4-D map)
      auto load_tile = [&](const CUtensorMap* tm, int y, int zc) {
        const uint32_t slot = seq % NS;
        ok = ok && mbar_wait(BAR(C::B_EMPTY + slot), ((seq / NS) & 1) ^ 1, abort);
        if (!ok) return;
        mbar_arrive_expect_tx(BAR(C::B_FULL + slot), C::TILE_BYTES);
        for (int b = 0; b < C::NBOX; ++b) {
          const uint32_t dst = ring + slot * C::TILE_BYTES + b * C::BOX_BYTES;
          if (zc >= 0)
            tma_load_3d(dst, tm, BAR(C::B_FULL + slot), 64 * b, y, zc);
          else
            tma_load_4d(dst, tm, BAR(C::B_FULL + slot), 64 * b, y, hh, bb);
        }
        ++seq;
      };
      for (int j = 0; j < ntiles && ok; ++j) {
        load_tile(&p.tm_k, lo + 128 * j, -1);
        load_tile(&p.tm_v, lo + 128 * j, -1);
      }
      if (has_lin) {
        // The bf16 hi/lo state tiles come from the kernel before this one
        // (launched with a programmatic dependency in the recurrent step).
        grid_dep_wait();
        const int zc = bh * p.state_mul + (p.g.step ? 0 : t);
        for (int part = 0; part < 2 && ok; ++part)
          for (int rr = 0; rr < C::SPP && ok; ++rr) load_tile(part ? &p.tm_lo : &p.tm_hi, 128 * rr, zc);
      }
      // drain: every copy issued must have landed before the CTA exits
      drain_wait(BAR(C::B_Q), 0);
      for (uint32_t s2 = (seq > NS ? seq - NS : 0); s2 < seq; ++s2) drain_wait(BAR(C::B_FULL + s2 % NS), (s2 / NS) & 1);
    }
  } else if (warp == 9) {
    // =============================== MMA issuer ==============================
    if (lane == 0) {
      const uint32_t qA = smem_u32(smem + C::OFF_Q);
      const uint32_t qB = qA + C::TILE_BYTES;
      const uint32_t ring = smem_u32(smem + C::OFF_RING);
      auto slot_addr = [&](uint32_t sq) { return ring + (sq % NS) * C::TILE_BYTES; };
      // Q K^T: A = Q tile, B = K tile, both K-major; K-step kk moves 32 B
      // inside a 128-B swizzle row (box kk/4).  Descriptors: constant high
      // word, low word = base + compile-time step (see desc_hi_sw128).
      constexpr uint32_t HI_K = desc_hi_sw128(1024);    // K-major: SBO = 8 rows
      constexpr uint32_t HI_MN = desc_hi_sw128(1024);   // MN-major: SBO = 8 K-rows
      const uint32_t lo_qA = desc_lo(qA, 16), lo_qB = desc_lo(qB, 16);
      auto issue_S = [&](uint32_t d_tmem, uint32_t lo_q, uint32_t kb) {
        const uint32_t lo_k = desc_lo(kb, 16);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t step = ((kk >> 2) * C::BOX_BYTES + (kk & 3) * 32) >> 4;
          mma_ss(d_tmem, desc_join(lo_q + step, HI_K), desc_join(lo_k + step, HI_K), C::IDESC_S, kk > 0 ? 1u : 0u);
        }
      };
      // P V: A = P in TMEM (8 columns per 16 keys), B = V tile MN-major:
      // 16 keys = 2048 B; the two 64-column boxes are BOX_BYTES apart (LBO).
      auto issue_PV_half = [&](uint32_t d_tmem, uint32_t a_tmem, uint32_t vb, bool first, int half) {
        const uint32_t lo_v = desc_lo(vb, C::BOX_BYTES);
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) {
          const int kk = 4 * half + k4;
          mma_ts(d_tmem, a_tmem + kk * 8, desc_join(lo_v + ((kk * 2048) >> 4), HI_MN), C::IDESC_PV,
                 (first && kk == 0) ? 0u : 1u);
        }
      };
      // O_X += P_X V_j, each 64-key half once the softmax warps have
      // released it
      auto issue_PV = [&](int X, uint32_t vb, int j) -> bool {
        if (!mbar_wait(BAR(C::B_P + X), j & 1, abort)) return false;
        TRACE(10 + X, j);
        tc_fence_after();
        issue_PV_half(tmem + 256 + X * D, tmem + X * 128, vb, j == 0, 0);
        if (!mbar_wait(BAR(C::B_P1 + X), j & 1, abort)) return false;
        tc_fence_after();
        issue_PV_half(tmem + 256 + X * D, tmem + X * 128, vb, j == 0, 1);
        return true;
      };
      TRACE(14, 0);
      bool ok = mbar_wait(BAR(C::B_Q), 0, abort);
      ok = ok && mbar_wait(BAR(C::B_FULL + 0), 0, abort);  // K_0 is sequence 0
      TRACE(14, 1);
      tc_fence_after();
      if (ok) {
        issue_S(tmem + 0, lo_qA, slot_addr(0));
        mma_commit(BAR(C::B_S + 0));
        if (hasB) {
          issue_S(tmem + 128, lo_qB, slot_addr(0));
          mma_commit(BAR(C::B_S + 1));
        }
        mma_commit(BAR(C::B_EMPTY + 0));
      }
      for (int j = 0; ok && j < ntiles; ++j) {
        const uint32_t vq = 2 * j + 1, kn = 2 * j + 2;
        const bool more = j + 1 < ntiles;
        ok = mbar_wait(BAR(C::B_FULL + vq % NS), (vq / NS) & 1, abort) && issue_PV(0, slot_addr(vq), j);
        if (!ok) break;
        mma_commit(BAR(C::B_PVD + 0));
        TRACE(15, j);
        if (more) {
          // S_A(j+1) = Q_A K_{j+1}^T overwrites the TMEM columns P_A(j) occupies,
          // the A operand of P_A(j) V_j: it is issued only once that MMA has
          // completed (its commit), as tcgen05 operands must not be modified
          // while an MMA that reads them is in flight.
          ok = mbar_wait(BAR(C::B_FULL + kn % NS), (kn / NS) & 1, abort) &&
               mbar_wait(BAR(C::B_PVD + 0), j & 1, abort);
          if (!ok) break;
          TRACE(14, j + 2);
          tc_fence_after();
          issue_S(tmem + 0, lo_qA, slot_addr(kn));
          mma_commit(BAR(C::B_S + 0));
          TRACE(12, j);
        } else {
          mma_commit(BAR(C::B_O + 0));
        }
        if (hasB) {
          ok = issue_PV(1, slot_addr(vq), j);
          if (!ok) break;
          mma_commit(BAR(C::B_EMPTY + vq % NS));
          mma_commit(BAR(C::B_PVD + 1));
          if (more) {
            ok = mbar_wait(BAR(C::B_PVD + 1), j & 1, abort);  // P_B(j) V_j complete (see S_A)
            if (!ok) break;
            tc_fence_after();
            issue_S(tmem + 128, lo_qB, slot_addr(kn));
            mma_commit(BAR(C::B_S + 1));
            TRACE(13, j);
            mma_commit(BAR(C::B_EMPTY + kn % NS));
          } else {
            mma_commit(BAR(C::B_O + 1));
          }
        } else {
          mma_commit(BAR(C::B_EMPTY + vq % NS));
          if (more) mma_commit(BAR(C::B_EMPTY + kn % NS));
        }
      }
      if (ok && has_lin) {
        // O += phi~(Q) [S_hi ; S_lo]: A = scaled phi(Q) in TMEM over the S
        // columns, B = state rows (features) x D, MN-major, 128 rows a slot.
        const uint32_t s0 = 2 * ntiles;
        for (int i = 0; i < 2 * C::SPP && ok; ++i)
          ok = mbar_wait(BAR(C::B_FULL + (s0 + i) % NS), ((s0 + i) / NS) & 1, abort);
        for (int X = 0; X < (hasB ? 2 : 1) && ok; ++X) {
          ok = mbar_wait(BAR(C::B_PHI + X), 0, abort);
          if (!ok) break;
          tc_fence_after();
          for (int part = 0; part < 2; ++part) {
#pragma unroll
            for (int kk = 0; kk < (2 * D) / 16; ++kk) {
              const uint32_t sa = slot_addr(s0 + part * C::SPP + kk / 8);
              const uint32_t acc = PARTS ? ((part | kk) != 0 ? 1u : 0u) : 1u;
              mma_ts(tmem + 256 + X * D, tmem + X * 128 + kk * 8,
                     desc_join(desc_lo(sa + (kk & 7) * 2048, C::BOX_BYTES), HI_MN), C::IDESC_PV, acc);
            }
          }
          mma_commit(BAR(C::B_LIN + X));
        }
        if (ok)
          for (int i = 0; i < 2 * C::SPP; ++i) mma_commit(BAR(C::B_EMPTY + (s0 + i) % NS));
      }
      // drain: all MMAs complete before TMEM is released
      mma_commit(BAR(C::B_FIN));
      drain_wait(BAR(C::B_FIN), 0);
    }
  }
#undef BAR
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace

int attn_smem_bytes(int D) { return D == 128 ? AttnCfg<128>::SMEM : AttnCfg<64>::SMEM; }

template <int D, bool PARTS, bool PHI = false>
static cudaError_t launch_attn_t(const AttnParams& p, int n_units, cudaStream_t s, bool pdl) {
  auto* k = hybrid_chunk_attn_kernel<D, PARTS, PHI>;
  // The in-kernel register split assumes exactly REGS_LAUNCH registers per
  // thread at launch; with fewer, a warpgroup's increase could never be met.
  cudaError_t e = prepare_kernel_once(reinterpret_cast<const void*>(k), AttnCfg<D>::SMEM,
                                      static_cast<int>(AttnCfg<D>::REGS_LAUNCH));
  if (e != cudaSuccess) return e;
  return launch_k(k, dim3(n_units), dim3(AttnCfg<D>::THREADS), AttnCfg<D>::SMEM, s, pdl, p);
}

cudaError_t launch_attention(int D, bool parts, const AttnParams& p, int n_units, cudaStream_t s, bool pdl) {
  if (n_units <= 0) return cudaSuccess;
  if (D == 128)
    return parts ? launch_attn_t<128, true>(p, n_units, s, pdl) : launch_attn_t<128, false>(p, n_units, s, pdl);
  return parts ? launch_attn_t<64, true>(p, n_units, s, pdl) : launch_attn_t<64, false>(p, n_units, s, pdl);
}

cudaError_t launch_attention_phi(int D, const AttnParams& p, int n_units, cudaStream_t s, bool pdl) {
  if (n_units <= 0) return cudaSuccess;
  return D == 128 ? launch_attn_t<128, false, true>(p, n_units, s, pdl)
                  : launch_attn_t<64, false, true>(p, n_units, s, pdl);
}

}  // namespace rehyat

namespace rehyat {
cudaError_t read_and_clear_device_error(unsigned int* v) {
  cudaError_t e = cudaMemcpyFromSymbol(v, g_device_error, sizeof(unsigned int));
  if (e != cudaSuccess) return e;
  const unsigned int zero = 0;
  return cudaMemcpyToSymbol(g_device_error, &zero, sizeof(unsigned int));
}
}  // namespace rehyat
