// geom.cuh -- chunk / segment geometry of ReHyAt's temporally chunked hybrid
// attention, shared by the host planner and the kernels.
//
// "ReHyAt: Recurrent Hybrid Attention for Video Diffusion Transformers",
// §3.3 (Recurrent HyAt): for chunk t,
//   T^S_t = { lo_t <= j < (t+1)N' },  T^L_t = { j < lo_t },
//   lo_t  = max(tN' - T_o HW, 0),
// with N' = T_c * HW tokens per chunk (chunk t owns queries [tN', (t+1)N'))
// and every range clipped to the N = F * HW tokens of the video.
//
// The linear state entering chunk t is the sum over [0, lo_t).  It is built
// from "segments": segment s covers keys [lo_s, lo_{s+1}), so the state of
// chunk t is the exclusive prefix over segments 0 .. t-1.
//
// With the §3.2 bidirectional sets (T^L_t = T - T^S_t) the state of chunk t
// is the sum over every key outside [lo_t, hi_t); segments are then single
// frames and the state is prefix(lo_t) + suffix(hi_t).
#pragma once

#include <cstdint>

namespace rehyat {

#if defined(__CUDACC__)
#define RH_HD __host__ __device__ __forceinline__
#else
#define RH_HD inline
#endif

RH_HD int imin(int a, int b) { return a < b ? a : b; }
RH_HD int imax(int a, int b) { return a > b ? a : b; }
RH_HD int cdiv(int a, int b) { return (a + b - 1) / b; }

// Query rows and softmax window of each chunk.  Two framings:
//  - parallel form: q and k/v are the whole video (N_q == N_k == N);
//  - step form: one chunk, q holds its queries [0, N_q) and k/v its whole
//    window [0, N_k) (overlap frames followed by the chunk's own frames).
struct ChunkGeom {
  int N_q;        // rows per (b,h) of the q / out tensors
  int N_k;        // rows per (b,h) of the k / v tensors
  int chunk_tok;  // N' = T_c * S_tok (parallel); N_q (step)
  int ovl_tok;    // T_o * S_tok (parallel); unused (step)
  int n_chunks;   // ceil(F / T_c) (parallel); 1 (step)
  int step;       // 0 = parallel framing, 1 = step framing

  RH_HD void chunk(int t, int& q0, int& q1, int& lo, int& hi) const {
    if (step) {
      q0 = 0; q1 = N_q; lo = 0; hi = N_k;
      return;
    }
    q0 = t * chunk_tok;
    q1 = imin(q0 + chunk_tok, N_q);
    lo = imax(q0 - ovl_tok, 0);
    hi = q1;
  }
};

// Key segments whose phi(K)^T V sums make up the linear states.
struct SegGeom {
  int N_k;        // rows per (b,h) of k / v
  int chunk_tok;  // N'
  int ovl_tok;    // T_o * S_tok
  int n_seg;      // number of segments (n_chunks - 1 in the parallel form; 1 in the step form)
  int nsplit;     // CTAs per segment (token ranges split evenly)
  int step;       // 1: a single segment [0, step_tok)
  int step_tok;
  int seg_tok;    // > 0: fixed segments [s * seg_tok, (s + 1) * seg_tok) (one frame each)

  RH_HD void seg(int s, int& a, int& b) const {
    if (step) {
      a = 0; b = step_tok;
      return;
    }
    if (seg_tok > 0) {
      a = imin(s * seg_tok, N_k);
      b = imin(a + seg_tok, N_k);
      return;
    }
    a = imin(imax(s * chunk_tok - ovl_tok, 0), N_k);
    b = imin(imax((s + 1) * chunk_tok - ovl_tok, 0), N_k);
  }
  RH_HD void piece(int s, int p, int& a, int& b) const {
    int sa, sb;
    seg(s, sa, sb);
    const int per = cdiv(sb - sa, nsplit);
    a = imin(sa + p * per, sb);
    b = imin(a + per, sb);
  }
};

}  // namespace rehyat
