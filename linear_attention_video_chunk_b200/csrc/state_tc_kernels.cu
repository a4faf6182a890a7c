// state_tc_kernels.cu -- phi_state_kernel: phi(K)^T V and sum phi(K) per key
// segment on the tensor cores (tcgen05 / TMEM / TMA) for sm_100a: the two
// query-independent sums of "ReHyAt: Recurrent Hybrid Attention for Video
// Diffusion Transformers" §3.1, with phi of §3.2 (P = 2, psi = 1 + elu) or a
// precomputed phi(K) of a learned map (§4.3, §7.1).
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

// ============================================================================
// Segment states: phi(K)^T V and sum phi(K)
// ============================================================================
template <int D, bool PRE>
struct StCfg {
  static constexpr int NBOX = D / 64;
  static constexpr int BOX = 64 * 128;                // 64 token rows x 128 B
  static constexpr int KV_BYTES = NBOX * BOX;         // 64 x D bf16
  static constexpr int PHI_BYTES = 2 * NBOX * BOX;    // 64 x 2D bf16
  // A ring stage holds K then V; phi(K) is computed into a separate two-deep
  // ring, so the ring's bytes go to loads in flight.  With phi(K)
  // precomputed a stage holds V then the phi(K) tile itself.
  static constexpr int STAGE = PRE ? KV_BYTES + PHI_BYTES : 2 * KV_BYTES;
  static constexpr int OFF_V = PRE ? 0 : KV_BYTES;    // V inside a stage
  static constexpr int OFF_PT = KV_BYTES;             // the phi(K) tile inside a stage (PRE)
  static constexpr int NST = PRE ? ((D == 128) ? 4 : 6) : ((D == 128) ? 5 : 8);
  static constexpr int NPHI = PRE ? 0 : 2;
  static constexpr int OFF_PHI = NST * STAGE;         // phi(K) ring (computed phi only)
  static constexpr int DATA = OFF_PHI + NPHI * PHI_BYTES;
  static constexpr int OFF_BAR = DATA;
  static constexpr int SMEM = OFF_BAR + 256 + 1024;
  static constexpr int HALVES = (2 * D) / 128;        // M = 128 feature blocks
  static constexpr uint32_t TMEM_COLS = (HALVES * D <= 64) ? 64 : ((HALVES * D <= 128) ? 128 : 256);
  static constexpr int PHI_WARPS = 16;                // warps 0-15: phi(K), sum phi(K), epilogue
                                                      // (four a sub-partition, to hide latency)
  static constexpr int PHI_THREADS = 32 * PHI_WARPS;
  static constexpr int THREADS = PHI_THREADS + 64;    // + TMA producer (warp 16) + MMA issuer (warp 17)
  static constexpr int CH = D / 8;                    // 16-byte chunks per row
  static constexpr int G = PHI_THREADS / CH;          // token groups
  static constexpr int TPG = 64 / G;                  // tokens per thread per tile
  // barriers: stage full / empty, phi buffer written / consumed by the MMA
  static constexpr int B_FULL = 0, B_EMPTY = NST, B_PHI = 2 * NST, B_PHIE = 2 * NST + 2;
  static constexpr int B_ACC = 2 * NST + 4, B_FIN = 2 * NST + 5;
  static_assert((B_FIN + 1) * 8 <= 224, "barrier area");
  // epilogue, over the drained ring: the 2D x D accumulators staged as fp32
  // rows of SROW bytes (D + 4 floats: rows 4 banks apart), then the
  // token-group partial sums of phi(K)
  static constexpr int SROW = (D + 4) * 4;
  static constexpr int OFF_ZRED = 2 * D * SROW;
  // A = phi(K)^T (features x tokens, features contiguous: MN-major),
  // B = V (tokens x D, D contiguous: MN-major).
  static constexpr uint32_t IDESC = idesc_bf16_f32(128, D, 1, 1);
  static_assert(SMEM <= 232448, "shared memory");
  static_assert(G * CH == PHI_THREADS && TPG * G == 64, "thread mapping");
  static_assert(OFF_ZRED + G * 2 * D * 4 <= DATA, "epilogue scratch");
  static_assert(2 * D <= PHI_THREADS, "one staged row a phi thread");
};

// PRE: phi(K) is precomputed (a learned feature map) and arrives by TMA
// through p.tm_phik straight into the A-operand layout; the phi warps then
// only zero the rows past the piece's end and sum phi(K).
template <int D, bool PRE>
__global__ void __launch_bounds__(StCfg<D, PRE>::THREADS, 1) phi_state_kernel(const __grid_constant__ StateParams p) {
  using C = StCfg<D, PRE>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  grid_dep_launch();  // the recurrent step's state update may be scheduled
  const int u = blockIdx.x;  // (bh * n_seg + s) * nsplit + piece
  const int piece = u % p.sg.nsplit;
  const int s = (u / p.sg.nsplit) % p.sg.n_seg;
  const int bh = u / (p.sg.nsplit * p.sg.n_seg);
  int a, b;
  p.sg.piece(s, piece, a, b);
  const int ntiles = cdiv(b - a, 64);
  float* outS = p.part_S + static_cast<size_t>(u) * (2 * D) * D;
  float* outz = p.part_z + static_cast<size_t>(u) * (2 * D);
  if (ntiles == 0) {  // empty piece: its sums are zero
    for (int i = threadIdx.x; i < 2 * D * D; i += blockDim.x) outS[i] = 0.f;
    for (int i = threadIdx.x; i < 2 * D; i += blockDim.x) outz[i] = 0.f;
    grid_dep_wait();
    return;
  }

  uint8_t* barea = smem + C::OFF_BAR;
  const uint32_t bar0 = smem_u32(barea);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(barea + 224);
  volatile int* abort = reinterpret_cast<volatile int*>(barea + 228);
#define BAR(i) (bar0 + 8u * static_cast<uint32_t>(i))
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NST; ++i) {
      mbar_init(BAR(C::B_FULL + i), 1);
      mbar_init(BAR(C::B_EMPTY + i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(BAR(C::B_PHI + i), C::PHI_WARPS);
      mbar_init(BAR(C::B_PHIE + i), 1);
    }
    mbar_init(BAR(C::B_ACC), 1);
    mbar_init(BAR(C::B_FIN), 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == C::PHI_WARPS && lane == 0) {
    if (PRE)
      prefetch_tmap(&p.tm_phik);
    else
      prefetch_tmap(&p.tm_k);
    prefetch_tmap(&p.tm_v);
  }
  if (warp == C::PHI_WARPS + 1) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < C::PHI_WARPS) {
    // ============ phi(K) into the MN-major A operand, sum phi(K) ============
    // phi atom bx (< NBOX) = psi of dims 64bx..64bx+63, atom NBOX+bx = psi^2:
    // byte-for-byte the same positions as the K box bx, so no re-layout.
    const int tid = threadIdx.x;
    const int c = tid % C::CH;
    const int g = tid / C::CH;
    const int bx = c >> 3, cc = c & 7;
    float za[8], zb[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) za[e] = zb[e] = 0.f;
    bool ok = true;
    for (int i = 0; i < ntiles; ++i) {
      const int st = i % C::NST;
      const int pb = i & 1;
      ok = mbar_wait(BAR(C::B_FULL + st), (i / C::NST) & 1, abort);
      // phi buffer pb is free once the MMA of tile i - 2 has completed
      if (ok && i >= 2) ok = mbar_wait(BAR(C::B_PHIE + pb), ((i >> 1) - 1) & 1, abort);
      if (!ok) break;
      const uint8_t* kt = smem + st * C::STAGE;
      uint8_t* ph = PRE ? smem + st * C::STAGE + C::OFF_PT : smem + C::OFF_PHI + pb * C::PHI_BYTES;
#pragma unroll
      for (int ii = 0; ii < C::TPG; ++ii) {
        const int tok = g + ii * C::G;
        const bool valid = a + 64 * i + tok < b;
        const int off = tok * 128 + ((cc ^ (tok & 7)) << 4);
        uint4 pa = make_uint4(0u, 0u, 0u, 0u), pb4 = pa;
        if (PRE) {
          uint4* fa = reinterpret_cast<uint4*>(ph + bx * C::BOX + off);
          uint4* fb = reinterpret_cast<uint4*>(ph + (C::NBOX + bx) * C::BOX + off);
          if (valid) {
            pa = *fa;
            pb4 = *fb;
            const uint32_t va[4] = {pa.x, pa.y, pa.z, pa.w};
            const uint32_t vb[4] = {pb4.x, pb4.y, pb4.z, pb4.w};
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              za[2 * h] = add_bf16_lo(va[h], za[2 * h]);
              za[2 * h + 1] = add_bf16_hi(va[h], za[2 * h + 1]);
              zb[2 * h] = add_bf16_lo(vb[h], zb[2 * h]);
              zb[2 * h + 1] = add_bf16_hi(vb[h], zb[2 * h + 1]);
            }
          } else {  // a later segment's token: out of this piece's sums
            *fa = pa;
            *fb = pb4;
          }
          continue;
        }
        if (valid) {
          const uint4 raw = *reinterpret_cast<const uint4*>(kt + bx * C::BOX + off);
          const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
          uint32_t va[4], vb[4];
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const float s0 = psi1(bf16lo(w[h])), s1 = psi1(bf16hi(w[h]));
            va[h] = pack_bf16(s0, s1);
            vb[h] = pack_bf16(s0 * s0, s1 * s1);
            // sum phi(K) over the same bf16 features the phi(K)^T V MMA uses
            za[2 * h] = add_bf16_lo(va[h], za[2 * h]);
            za[2 * h + 1] = add_bf16_hi(va[h], za[2 * h + 1]);
            zb[2 * h] = add_bf16_lo(vb[h], zb[2 * h]);
            zb[2 * h + 1] = add_bf16_hi(vb[h], zb[2 * h + 1]);
          }
          pa = make_uint4(va[0], va[1], va[2], va[3]);
          pb4 = make_uint4(vb[0], vb[1], vb[2], vb[3]);
        }
        *reinterpret_cast<uint4*>(ph + bx * C::BOX + off) = pa;
        *reinterpret_cast<uint4*>(ph + (C::NBOX + bx) * C::BOX + off) = pb4;
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(C::B_PHI + pb));
    }
    // ---- epilogue: TMEM accumulators -> partial state rows ----
    // Every MMA has completed once B_ACC fires, so the ring is drained and
    // serves as the staging area: rows go to shared memory at a padded
    // stride, then out by contiguous bulk copies (one 4D-byte row each).
    if (ok) ok = mbar_wait(BAR(C::B_ACC), 0, abort);
    ok = __all_sync(kFull, ok);
    tc_fence_after();
    // warps w, w+4, w+8, w+12 cover the same TMEM lanes; with two feature
    // halves they split the work by half and by column half, with one
    // (D = 64) the first two take 32 columns each and the others none
    const int quarter = warp & 3, grp = warp >> 2;
    const int h = (C::HALVES == 2) ? (grp & 1) : 0;
    constexpr int NCOL = (C::HALVES == 2) ? D / 2 : 32;
    const int col0 = (C::HALVES == 2) ? (grp >> 1) * (D / 2) : grp * 32;
    if (ok && col0 < D) {
      const int e = 128 * h + 32 * quarter + lane;
#pragma unroll
      for (int q = 0; q < NCOL / 32; ++q) {
        uint32_t v[32];
        tmem_ld32(tmem + (static_cast<uint32_t>(32 * quarter) << 16) + h * D + col0 + 32 * q, v);
        tmem_ld_wait();
        reg_fence(v);
        float4* dst = reinterpret_cast<float4*>(smem + e * C::SROW + (col0 + 32 * q) * 4);
#pragma unroll
        for (int k4 = 0; k4 < 8; ++k4)
          dst[k4] = make_float4(__uint_as_float(v[4 * k4]), __uint_as_float(v[4 * k4 + 1]),
                                __uint_as_float(v[4 * k4 + 2]), __uint_as_float(v[4 * k4 + 3]));
      }
    }
    // sum phi(K) across the token groups (the barrier is reached by every
    // phi thread whatever `ok` is)
    float* zred = reinterpret_cast<float*>(smem + C::OFF_ZRED);
    if (ok) {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        zred[g * 2 * D + 8 * c + e] = za[e];
        zred[g * 2 * D + D + 8 * c + e] = zb[e];
      }
    }
    fence_proxy_async_smem();  // the staged rows are read by the bulk copies
    asm volatile("bar.sync 1, %0;" ::"n"(C::PHI_THREADS) : "memory");
    if (ok && tid < 2 * D) {
      // one staged row a thread: a contiguous 4D-byte copy
      bulk_store(outS + static_cast<size_t>(tid) * D, smem_u32(smem) + tid * C::SROW, D * 4);
      bulk_commit();
      float acc = 0.f;
      for (int gg = 0; gg < C::G; ++gg) acc += zred[gg * 2 * D + tid];
      outz[tid] = acc;
      bulk_wait<0>();  // the row is written (and the staging area read) before exit
    }
  } else if (warp == C::PHI_WARPS) {
    // =============================== TMA producer ============================
    if (lane == 0) {
      bool ok = true;
      int i = 0;
      for (; i < ntiles && ok; ++i) {
        const int st = i % C::NST;
        ok = mbar_wait(BAR(C::B_EMPTY + st), ((i / C::NST) & 1) ^ 1, abort);
        if (!ok) break;
        const uint32_t base = smem_u32(smem + st * C::STAGE);
        mbar_arrive_expect_tx(BAR(C::B_FULL + st), C::STAGE);
        for (int bb = 0; bb < C::NBOX; ++bb) {
          if (!PRE)
            tma_load_4d(base + bb * C::BOX, &p.tm_k, BAR(C::B_FULL + st), 64 * bb, a + 64 * i, bh % p.H, bh / p.H);
          tma_load_4d(base + C::OFF_V + bb * C::BOX, &p.tm_v, BAR(C::B_FULL + st), 64 * bb, a + 64 * i, bh % p.H,
                      bh / p.H);
        }
        if (PRE)
          for (int bb = 0; bb < 2 * C::NBOX; ++bb)
            tma_load_4d(base + C::OFF_PT + bb * C::BOX, &p.tm_phik, BAR(C::B_FULL + st), 64 * bb, a + 64 * i,
                        bh % p.H, bh / p.H);
      }
      for (int i2 = (i > C::NST ? i - C::NST : 0); i2 < i; ++i2)
        drain_wait(BAR(C::B_FULL + i2 % C::NST), (i2 / C::NST) & 1);
    }
  } else {
    // =============================== MMA issuer ==============================
    if (lane == 0) {
      bool ok = true;
      for (int i = 0; i < ntiles && ok; ++i) {
        const int st = i % C::NST;
        const int pb = i & 1;
        ok = mbar_wait(BAR(C::B_FULL + st), (i / C::NST) & 1, abort) &&
             mbar_wait(BAR(C::B_PHI + pb), (i >> 1) & 1, abort);
        if (!ok) break;
        tc_fence_after();
        const uint32_t vb = smem_u32(smem + st * C::STAGE + C::OFF_V);
        const uint32_t pbase =
            PRE ? smem_u32(smem + st * C::STAGE + C::OFF_PT) : smem_u32(smem + C::OFF_PHI + pb * C::PHI_BYTES);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {  // 16 tokens per MMA
#pragma unroll
          for (int h = 0; h < C::HALVES; ++h)
            mma_ss(tmem + h * D, smem_desc_sw128(pbase + 2 * h * C::BOX + kk * 2048, C::BOX, 1024),
                   smem_desc_sw128(vb + kk * 2048, C::BOX, 1024), C::IDESC, (i > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(BAR(C::B_EMPTY + st));
        mma_commit(BAR(C::B_PHIE + pb));
      }
      if (ok) mma_commit(BAR(C::B_ACC));
      mma_commit(BAR(C::B_FIN));
      drain_wait(BAR(C::B_FIN), 0);
    }
  }
#undef BAR
  tc_fence_before();
  __syncthreads();
  if (warp == C::PHI_WARPS + 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
  // Launched behind the recurrent step's attention with a programmatic
  // dependency (it reads only the chunk's keys and values): it completes only
  // after that attention has, so the state update launched next may rely on
  // both.  Launched normally, this returns at once.
  grid_dep_wait();
}

// Failure-path check: one warp waits on an mbarrier that nothing ever
// arrives on.  The bounded wait gives up after its limit, records the timeout
// in this unit's device error word and returns, so the host reads
// REHYAT_ETIMEOUT and the context stays usable.
__global__ void wait_probe_kernel(int* gave_up) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_word;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_word = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const bool ok = mbar_wait(smem_u32(&bar), 0, &abort_word);
  if (threadIdx.x == 0 && gave_up != nullptr) *gave_up = ok ? 0 : 1;
}

}  // namespace

cudaError_t launch_wait_probe(int* gave_up, cudaStream_t s) {
  wait_probe_kernel<<<1, 32, 0, s>>>(gave_up);
  return cudaGetLastError();
}

int state_smem_bytes(int D) {
  return D == 128 ? imax(StCfg<128, false>::SMEM, StCfg<128, true>::SMEM)
                  : imax(StCfg<64, false>::SMEM, StCfg<64, true>::SMEM);
}

template <int D, bool PRE = false>
static cudaError_t launch_state_t(const StateParams& p, int n_ctas, cudaStream_t s, bool pdl) {
  auto* k = phi_state_kernel<D, PRE>;
  using C = StCfg<D, PRE>;
  cudaError_t e = prepare_kernel_once(reinterpret_cast<const void*>(k), C::SMEM, 0);
  if (e != cudaSuccess) return e;
  return launch_k(k, dim3(n_ctas), dim3(C::THREADS), C::SMEM, s, pdl, p);
}

cudaError_t launch_chunk_state(int D, const StateParams& p, int n_ctas, cudaStream_t s, bool pdl) {
  if (n_ctas <= 0) return cudaSuccess;
  return D == 128 ? launch_state_t<128>(p, n_ctas, s, pdl) : launch_state_t<64>(p, n_ctas, s, pdl);
}

cudaError_t launch_chunk_state_phi(int D, const StateParams& p, int n_ctas, cudaStream_t s, bool pdl) {
  if (n_ctas <= 0) return cudaSuccess;
  return D == 128 ? launch_state_t<128, true>(p, n_ctas, s, pdl) : launch_state_t<64, true>(p, n_ctas, s, pdl);
}

cudaError_t read_and_clear_device_error_states(unsigned int* v) {
  cudaError_t e = cudaMemcpyFromSymbol(v, g_device_error, sizeof(unsigned int));
  if (e != cudaSuccess) return e;
  const unsigned int zero = 0;
  return cudaMemcpyToSymbol(g_device_error, &zero, sizeof(unsigned int));
}

}  // namespace rehyat
