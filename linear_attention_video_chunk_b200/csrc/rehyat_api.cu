// rehyat_api.cu -- the C ABI declared in include/rehyat.h: argument
// validation, scratch planning, TMA tensor maps and kernel launches.  No
// arithmetic of the method lives here.
#include <climits>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "geom.cuh"
#include "kernels.cuh"
#include "mlp.cuh"
#include "rehyat.h"

#define REHYAT_API extern "C" __attribute__((visibility("default")))

namespace rehyat {
cudaError_t read_and_clear_device_error(unsigned int* v);
cudaError_t read_and_clear_device_error_mlp(unsigned int* v);
cudaError_t read_and_clear_device_error_states(unsigned int* v);
cudaError_t launch_wait_probe(int* gave_up, cudaStream_t s);
}

namespace {
using namespace rehyat;

// CTAs aimed at for the state kernels: one wave of B200's 148 SMs (a
// constant, so the fp32 summation order does not depend on the device).
constexpr int kSplitTarget = 148;

// ---------------------------------------------------------------------------
// validation
// ---------------------------------------------------------------------------
int check_ptr(const void* p) {
  if (p == nullptr) return REHYAT_EINVAL;
  if (reinterpret_cast<uintptr_t>(p) % 16 != 0) return REHYAT_EINVAL;
  return REHYAT_OK;
}

int check_d(int d) {
  if (d < 1) return REHYAT_EINVAL;
  if (d != 64 && d != 128) return REHYAT_EUNSUPPORTED;
  return REHYAT_OK;
}

// ---------------------------------------------------------------------------
// plans
// ---------------------------------------------------------------------------
size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct FwdPlan {
  int BH, N, D, nc, n_seg, nsplit, chunk_tok, ovl_tok, pairs, n_units;
  int F, S_tok, tc, to, bidir;  // bidir: §3.2 sets (frame segments, prefix + suffix states)
  int B, H;
  long long rs, hs, bs;         // q/k/v/out element strides of a row, a head, a batch
  size_t off_pS, off_pz, off_hi, off_lo, off_zt, bytes;       // bf16 path
  size_t f32_off_pS, f32_off_pz, f32_off_S, f32_off_zt, f32_bytes;  // fp32 path
};

int plan_forward(int B, int H, int F, int S_tok, int d, int Tc, int To, FwdPlan* p) {
  if (B < 1 || H < 1 || F < 1 || S_tok < 1 || Tc < 1 || To < 0) return REHYAT_EINVAL;
  int st = check_d(d);
  if (st != REHYAT_OK) return st;
  const long long BH = static_cast<long long>(B) * H;
  const long long N = static_cast<long long>(F) * S_tok;
  if (BH > INT_MAX || N > INT_MAX / 2) return REHYAT_EINVAL;
  if (BH * N * d > (1LL << 46)) return REHYAT_EINVAL;
  // A chunk (or an overlap) longer than the video is the whole video.
  const int tc = Tc < F ? Tc : F;
  const int to = To < F ? To : F;
  p->BH = static_cast<int>(BH);
  p->B = B;
  p->H = H;
  p->rs = d;                      // [B, H, N, d] unless a layout says otherwise
  p->hs = N * d;
  p->bs = H * N * d;
  p->N = static_cast<int>(N);
  p->D = d;
  p->F = F;
  p->S_tok = S_tok;
  p->tc = tc;
  p->to = to;
  p->bidir = 0;
  p->chunk_tok = tc * S_tok;
  p->ovl_tok = to * S_tok;
  p->nc = cdiv(F, tc);
  p->n_seg = p->nc - 1;
  const int max_tiles = cdiv(p->chunk_tok, 64);
  p->nsplit = 1;
  if (p->n_seg > 0) {  // pieces per segment: at most one wave of CTAs
    const long long want = kSplitTarget / (BH * p->n_seg);
    p->nsplit = static_cast<int>(want < 1 ? 1 : (want > max_tiles ? max_tiles : want));
  }
  p->pairs = cdiv(cdiv(p->chunk_tok, 128), 2);
  const long long units = BH * p->nc * static_cast<long long>(p->pairs);
  if (units > INT_MAX || BH * p->n_seg * static_cast<long long>(p->nsplit) > INT_MAX) return REHYAT_EINVAL;
  p->n_units = static_cast<int>(units);
  const size_t D2 = 2 * static_cast<size_t>(d);
  const size_t segs = static_cast<size_t>(BH) * p->n_seg * p->nsplit;
  const size_t chunks = static_cast<size_t>(BH) * p->nc;
  size_t off = 0;
  p->off_pS = off; off += align256(segs * D2 * d * 4);
  p->off_pz = off; off += align256(segs * D2 * 4);
  p->off_hi = off; off += align256(chunks * D2 * d * 2);
  p->off_lo = off; off += align256(chunks * D2 * d * 2);
  p->off_zt = off; off += align256(chunks * D2 * 4);
  p->bytes = off > 0 ? off : 256;
  const size_t segs1 = static_cast<size_t>(BH) * p->n_seg;
  off = 0;
  p->f32_off_pS = off; off += align256(segs1 * D2 * d * 4);
  p->f32_off_pz = off; off += align256(segs1 * D2 * 4);
  p->f32_off_S = off; off += align256(chunks * D2 * d * 4);
  p->f32_off_zt = off; off += align256(chunks * D2 * 4);
  p->f32_bytes = off;
  if (p->nc > 65535 || p->BH > 65535) p->f32_bytes = 0;  // fp32 grids use y/z dims
  return REHYAT_OK;
}

// Plan for the chosen sets.  The bidirectional sets sum keys per frame (so
// that both window edges are segment edges); the attention is unchanged.
int plan_forward_sets(int B, int H, int F, int S_tok, int d, int Tc, int To, int sets, FwdPlan* p) {
  if (sets != REHYAT_SETS_CAUSAL && sets != REHYAT_SETS_BIDIRECTIONAL) return REHYAT_EINVAL;
  int st = plan_forward(B, H, F, S_tok, d, Tc, To, p);
  if (st != REHYAT_OK || sets == REHYAT_SETS_CAUSAL) return st;
  p->bidir = 1;
  p->n_seg = (p->nc > 1) ? F : 0;  // one chunk: the complement of its window is empty
  p->nsplit = 1;
  if (p->n_seg > 0) {
    const long long want = kSplitTarget / (static_cast<long long>(p->BH) * p->n_seg);
    const int max_tiles = cdiv(S_tok, 64);
    p->nsplit = static_cast<int>(want < 1 ? 1 : (want > max_tiles ? max_tiles : want));
  }
  if (static_cast<long long>(p->BH) * p->n_seg * p->nsplit > INT_MAX) return REHYAT_EINVAL;
  const size_t D2 = 2 * static_cast<size_t>(d);
  const size_t segs = static_cast<size_t>(p->BH) * p->n_seg * p->nsplit;
  const size_t chunks = static_cast<size_t>(p->BH) * p->nc;
  size_t off = 0;
  p->off_pS = off; off += align256(segs * D2 * d * 4);
  p->off_pz = off; off += align256(segs * D2 * 4);
  p->off_hi = off; off += align256(chunks * D2 * d * 2);
  p->off_lo = off; off += align256(chunks * D2 * d * 2);
  p->off_zt = off; off += align256(chunks * D2 * 4);
  p->bytes = off > 0 ? off : 256;
  return REHYAT_OK;
}

// Element strides for a q/k/v/out layout.
int apply_layout(int layout, FwdPlan* p) {
  const long long N = p->N, d = p->D, H = p->H;
  if (layout == REHYAT_LAYOUT_BHND) {
    p->rs = d; p->hs = N * d; p->bs = H * N * d;
  } else if (layout == REHYAT_LAYOUT_BNHD) {
    p->rs = H * d; p->hs = d; p->bs = N * H * d;
  } else {
    return REHYAT_EINVAL;
  }
  return REHYAT_OK;
}

struct StepPlan {
  int B, H;
  int BH, D, Nq, Nk, evict_tok, nsplit, pairs, n_units;
  int split_begin, n_split;  // key-window split of the attention's last wave (AttnParams)
  size_t off_hi, off_lo, off_pS, off_pz, off_part, bytes;
  size_t f32_off_pS, f32_off_pz, f32_bytes;
};

int plan_step(int B, int H, int S_tok, int d, int qf, int cf, int ef, StepPlan* p) {
  if (B < 1 || H < 1 || S_tok < 1 || qf < 1 || cf < 0 || ef < 0) return REHYAT_EINVAL;
  int st = check_d(d);
  if (st != REHYAT_OK) return st;
  if (static_cast<long long>(ef) > static_cast<long long>(cf) + qf) return REHYAT_EINVAL;
  const long long BH = static_cast<long long>(B) * H;
  const long long Nq = static_cast<long long>(qf) * S_tok;
  const long long Nk = (static_cast<long long>(cf) + qf) * S_tok;
  if (BH > 65535 || Nk > INT_MAX / 2) return REHYAT_EINVAL;
  if (BH * Nk * d > (1LL << 46)) return REHYAT_EINVAL;
  p->BH = static_cast<int>(BH);
  p->B = B;
  p->H = H;
  p->D = d;
  p->Nq = static_cast<int>(Nq);
  p->Nk = static_cast<int>(Nk);
  p->evict_tok = ef * S_tok;
  const int max_tiles = cdiv(p->evict_tok > 0 ? p->evict_tok : 1, 64);
  const long long want = kSplitTarget / BH;
  p->nsplit = static_cast<int>(want < 1 ? 1 : (want > max_tiles ? max_tiles : want));
  p->pairs = cdiv(cdiv(p->Nq, 128), 2);
  const long long units = BH * p->pairs;
  if (units > INT_MAX) return REHYAT_EINVAL;
  p->n_units = static_cast<int>(units);
  // The attention's units are ordered pair-major, so the units with a
  // single query tile (the ragged last pair) come last.  When the units do
  // not fill a whole number of waves of kSplitTarget CTAs, the last full
  // units run as two CTAs over the two halves of the key window, as many as
  // fit beside the single-tile units in one last wave (needs >= 2 key tiles).
  {
    const int U = p->n_units;
    const int U_t = (cdiv(p->Nq, 128) % 2) ? p->BH : 0;
    const int R = U % kSplitTarget;
    int s_ = 0;
    if (U > kSplitTarget && R > 0 && cdiv(p->Nk, 128) >= 2) {
      s_ = imin(R - U_t, kSplitTarget - R);
      if (s_ < 0) s_ = 0;
    }
    p->n_split = s_;
    p->split_begin = (U - U_t) - s_;
  }
  const size_t D2 = 2 * static_cast<size_t>(d);
  size_t off = 0;
  p->off_hi = off; off += align256(static_cast<size_t>(BH) * D2 * d * 2);
  p->off_lo = off; off += align256(static_cast<size_t>(BH) * D2 * d * 2);
  p->off_pS = off; off += align256(static_cast<size_t>(BH) * p->nsplit * D2 * d * 4);
  p->off_pz = off; off += align256(static_cast<size_t>(BH) * p->nsplit * D2 * 4);
  p->off_part = off; off += align256(static_cast<size_t>(p->n_split) * 2 * 2 * 128 * (d + 4) * 4);
  p->bytes = off;
  off = 0;
  p->f32_off_pS = off; off += align256(static_cast<size_t>(BH) * D2 * d * 4);
  p->f32_off_pz = off; off += align256(static_cast<size_t>(BH) * D2 * 4);
  p->f32_bytes = off;
  return REHYAT_OK;
}

// ---------------------------------------------------------------------------
// TMA tensor maps (driver entry point fetched through the runtime, so the
// library does not link libcuda directly)
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  });
  return fn;
}

// bf16 tensor [depth, rows, inner] (inner fastest), boxes of 64 x box_rows,
// 128-byte swizzle, zero fill out of bounds.
bool make_map(CUtensorMap* m, const void* base, long long inner, long long rows, long long depth, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(depth)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(inner) * 2, static_cast<cuuint64_t>(inner) * 2 * rows};
  cuuint32_t box[3] = {64u, static_cast<cuuint32_t>(box_rows), 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 tensor of B x H x rows x inner with arbitrary element strides for a
// row, a head and a batch (inner is contiguous): 4-D map {inner, rows, H, B},
// boxes of 64 x box_rows x 1 x 1, 128-byte swizzle, zero fill out of bounds.
bool make_map4(CUtensorMap* m, const void* base, long long inner, long long rows, long long H, long long B,
               long long rs, long long hs, long long bs, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(H),
                        static_cast<cuuint64_t>(B)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(rs) * 2, static_cast<cuuint64_t>(hs) * 2,
                           static_cast<cuuint64_t>(bs) * 2};
  cuuint32_t box[4] = {64u, static_cast<cuuint32_t>(box_rows), 1u, 1u};
  cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? REHYAT_OK : REHYAT_ECUDA; }

#ifdef REHYAT_TRACE
unsigned long long* g_trace = nullptr;  // cycle-trace buffer of trace builds
#endif

// ---------------------------------------------------------------------------
// stages
// ---------------------------------------------------------------------------
// phi_k (optional): precomputed phi(K) [B, H, N, 2d] of a learned feature map.
int run_states(const void* k, const void* v, const FwdPlan& P, uint8_t* ws, float* Sf_out, float* z_out,
               cudaStream_t s, const void* phi_k = nullptr) {
  float* pS = reinterpret_cast<float*>(ws + P.off_pS);
  float* pz = reinterpret_cast<float*>(ws + P.off_pz);
  if (P.n_seg > 0) {
    StateParams sp;
    std::memset(&sp, 0, sizeof(sp));
    const long long D2 = 2LL * P.D;
    if ((phi_k == nullptr && !make_map4(&sp.tm_k, k, P.D, P.N, P.H, P.B, P.rs, P.hs, P.bs, 64)) ||
        (phi_k != nullptr &&
         !make_map4(&sp.tm_phik, phi_k, D2, P.N, P.H, P.B, D2, P.N * D2, P.H * P.N * D2, 64)) ||
        !make_map4(&sp.tm_v, v, P.D, P.N, P.H, P.B, P.rs, P.hs, P.bs, 64))
      return REHYAT_ECUDA;
    sp.sg = SegGeom{P.N, P.chunk_tok, P.ovl_tok, P.n_seg, P.nsplit, 0, 0, P.bidir ? P.S_tok : 0};
    sp.BH = P.BH;
    sp.H = P.H;
    sp.part_S = pS;
    sp.part_z = pz;
    const int n_ctas = P.BH * P.n_seg * P.nsplit;
    int st = cuda_status(phi_k != nullptr ? launch_chunk_state_phi(P.D, sp, n_ctas, s)
                                          : launch_chunk_state(P.D, sp, n_ctas, s));
    if (st != REHYAT_OK) return st;
  }
  if (P.bidir) {
    if (P.n_seg == 0)  // one chunk: no linear set; the causal scan writes zero states
      return cuda_status(launch_state_scan(pS, pz, P.BH, 0, 1, P.nc, P.D,
                                           Sf_out ? nullptr : reinterpret_cast<__nv_bfloat16*>(ws + P.off_hi),
                                           Sf_out ? nullptr : reinterpret_cast<__nv_bfloat16*>(ws + P.off_lo), Sf_out,
                                           Sf_out ? z_out : reinterpret_cast<float*>(ws + P.off_zt), s));
    return cuda_status(launch_state_scan_bidir(pS, pz, P.BH, P.F, P.nsplit, P.nc, P.D, P.tc, P.to,
                                               Sf_out ? nullptr : reinterpret_cast<__nv_bfloat16*>(ws + P.off_hi),
                                               Sf_out ? nullptr : reinterpret_cast<__nv_bfloat16*>(ws + P.off_lo),
                                               Sf_out, Sf_out ? z_out : reinterpret_cast<float*>(ws + P.off_zt), s));
  }
  if (Sf_out != nullptr)
    return cuda_status(launch_state_scan(pS, pz, P.BH, P.n_seg, P.nsplit, P.nc, P.D, nullptr, nullptr, Sf_out,
                                         z_out, s));
  return cuda_status(launch_state_scan(pS, pz, P.BH, P.n_seg, P.nsplit, P.nc, P.D,
                                       reinterpret_cast<__nv_bfloat16*>(ws + P.off_hi),
                                       reinterpret_cast<__nv_bfloat16*>(ws + P.off_lo), nullptr,
                                       reinterpret_cast<float*>(ws + P.off_zt), s));
}

// phi_q (optional): precomputed phi(q) [B, H, N, 2d] of a learned feature map.
int run_attention(const void* q, const void* k, const void* v, const FwdPlan& P, uint8_t* ws, void* out,
                  float* aS, float* nS, float* aL, float* nL, float* Mo, cudaStream_t s,
                  const void* phi_q = nullptr) {
  AttnParams ap;
  std::memset(&ap, 0, sizeof(ap));
  if (!make_map4(&ap.tm_q, q, P.D, P.N, P.H, P.B, P.rs, P.hs, P.bs, 128) ||
      !make_map4(&ap.tm_k, k, P.D, P.N, P.H, P.B, P.rs, P.hs, P.bs, 128) ||
      !make_map4(&ap.tm_v, v, P.D, P.N, P.H, P.B, P.rs, P.hs, P.bs, 128) ||
      !make_map(&ap.tm_hi, ws + P.off_hi, P.D, 2LL * P.D, static_cast<long long>(P.BH) * P.nc, 128) ||
      !make_map(&ap.tm_lo, ws + P.off_lo, P.D, 2LL * P.D, static_cast<long long>(P.BH) * P.nc, 128))
    return REHYAT_ECUDA;
  ap.g = ChunkGeom{P.N, P.N, P.chunk_tok, P.ovl_tok, P.nc, 0};
  ap.BH = P.BH;
  ap.H = P.H;
  ap.o_sb = P.bs;
  ap.o_sh = P.hs;
  ap.o_sr = P.rs;
  ap.pairs = P.pairs;
  ap.state_mul = P.nc;
  ap.scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(P.D));
  ap.z = reinterpret_cast<const float*>(ws + P.off_zt);
  ap.z_bh = 2LL * P.D * P.nc;
  ap.z_t = 2LL * P.D;
  ap.out = static_cast<__nv_bfloat16*>(out);
  ap.aS = aS; ap.nS = nS; ap.aL = aL; ap.nL = nL; ap.Mo = Mo;
#ifdef REHYAT_TRACE
  ap.trace = g_trace;
#endif
  if (phi_q != nullptr) {
    ap.phi_q = static_cast<const __nv_bfloat16*>(phi_q);
    return cuda_status(launch_attention_phi(P.D, ap, P.n_units, s));
  }
  return cuda_status(launch_attention(P.D, aS != nullptr, ap, P.n_units, s));
}

// Learned feature maps of up to two inputs (q then k) in one launch; every
// x is [B, N, H, d] or [B, H, N, d] by (rs, hs, bs), every phi [B, H, N, 2d].
struct MlpArgs {
  const void* x;
  const void* W1;
  const float* b1;
  const void* W2;
  const float* b2;
  void* phi;
};

int check_mlp_args(const MlpArgs& a) {
  if (check_ptr(a.x) || check_ptr(a.W1) || check_ptr(a.b1) || check_ptr(a.W2) || check_ptr(a.b2) ||
      check_ptr(a.phi))
    return REHYAT_EINVAL;
  return REHYAT_OK;
}

int run_phi_mlp(const MlpArgs* maps, int n_maps, int B, int H, int N, int d, long long rs, long long hs,
                long long bs, cudaStream_t s) {
  MlpParams mp;
  std::memset(&mp, 0, sizeof(mp));
  const long long D2 = 2LL * d;
  for (int i = 0; i < n_maps; ++i) {
    if (!make_map4(&mp.tm_x[i], maps[i].x, d, N, H, B, rs, hs, bs, 128) ||
        !make_map(&mp.tm_w1[i], maps[i].W1, d, D2, H, static_cast<int>(D2)) ||
        !make_map(&mp.tm_w2[i], maps[i].W2, D2, D2, H, static_cast<int>(D2)))
      return REHYAT_ECUDA;
    mp.b1[i] = maps[i].b1;
    mp.b2[i] = maps[i].b2;
    mp.phi[i] = static_cast<__nv_bfloat16*>(maps[i].phi);
  }
  mp.N = N;
  mp.H = H;
  mp.BH = B * H;
  // one wave of CTAs over the (map, bh) pairs, each walking its share of the
  // 128-row tiles with the head's weights loaded once
  const int pairs = n_maps * mp.BH;
  const int ntiles = cdiv(N, 128);
  int groups = kSplitTarget / pairs;
  groups = groups < 1 ? 1 : (groups > ntiles ? ntiles : groups);
  if (static_cast<long long>(pairs) * groups > INT_MAX) return REHYAT_EINVAL;
  mp.groups = groups;
#ifdef REHYAT_TRACE
  mp.trace = g_trace;
#endif
  return cuda_status(launch_phi_mlp(d, mp, n_maps, s));
}

struct WsGuard {  // stream-ordered scratch owned by one call
  void* p = nullptr;
  cudaStream_t s;
  explicit WsGuard(cudaStream_t st) : s(st) {}
  int alloc(size_t bytes) {
    if (cudaMallocAsync(&p, bytes > 0 ? bytes : 256, s) != cudaSuccess) {
      (void)cudaGetLastError();
      p = nullptr;
      return REHYAT_ENOMEM;
    }
    return REHYAT_OK;
  }
  ~WsGuard() {
    if (p != nullptr) (void)cudaFreeAsync(p, s);
  }
};

int check_qkvo(const void* q, const void* k, const void* v, const void* o) {
  int st = check_ptr(q);
  if (st == REHYAT_OK) st = check_ptr(k);
  if (st == REHYAT_OK) st = check_ptr(v);
  if (st == REHYAT_OK) st = check_ptr(o);
  return st;
}

}  // namespace

// ===========================================================================
// exported entry points
// ===========================================================================
REHYAT_API const char* rehyat_status_string(int status) {
  switch (status) {
    case REHYAT_OK: return "REHYAT_OK";
    case REHYAT_EINVAL: return "REHYAT_EINVAL: invalid argument";
    case REHYAT_EUNSUPPORTED: return "REHYAT_EUNSUPPORTED: unsupported configuration (d must be 64 or 128)";
    case REHYAT_ENOMEM: return "REHYAT_ENOMEM: workspace allocation failed or workspace too small";
    case REHYAT_ECUDA: return "REHYAT_ECUDA: CUDA call or kernel launch failed";
    case REHYAT_ETIMEOUT: return "REHYAT_ETIMEOUT: a bounded device-side wait ran out";
    default: return "REHYAT_UNKNOWN_STATUS";
  }
}

REHYAT_API int rehyat_forward_workspace_bytes(int B, int H, int F, int S_tok, int d, int chunk_frames,
                                              int overlap_frames, size_t* bytes) {
  if (bytes == nullptr) return REHYAT_EINVAL;
  FwdPlan P;
  int st = plan_forward(B, H, F, S_tok, d, chunk_frames, overlap_frames, &P);
  if (st != REHYAT_OK) return st;
  *bytes = P.bytes;
  return REHYAT_OK;
}

REHYAT_API int rehyat_forward_states(const void* k, const void* v, int B, int H, int F, int S_tok, int d,
                                     int chunk_frames, int overlap_frames, void* workspace,
                                     size_t workspace_bytes, void* stream) {
  FwdPlan P;
  int st = plan_forward(B, H, F, S_tok, d, chunk_frames, overlap_frames, &P);
  if (st != REHYAT_OK) return st;
  if (check_ptr(k) || check_ptr(v) || check_ptr(workspace)) return REHYAT_EINVAL;
  if (reinterpret_cast<uintptr_t>(workspace) % 256 != 0) return REHYAT_EINVAL;
  if (workspace_bytes < P.bytes) return REHYAT_ENOMEM;
  return run_states(k, v, P, static_cast<uint8_t*>(workspace), nullptr, nullptr, static_cast<cudaStream_t>(stream));
}

REHYAT_API int rehyat_forward_attention(const void* q, const void* k, const void* v, int B, int H, int F,
                                        int S_tok, int d, int chunk_frames, int overlap_frames, void* out,
                                        void* workspace, size_t workspace_bytes, void* stream) {
  FwdPlan P;
  int st = plan_forward(B, H, F, S_tok, d, chunk_frames, overlap_frames, &P);
  if (st != REHYAT_OK) return st;
  if (check_qkvo(q, k, v, out) || check_ptr(workspace)) return REHYAT_EINVAL;
  if (reinterpret_cast<uintptr_t>(workspace) % 256 != 0) return REHYAT_EINVAL;
  if (workspace_bytes < P.bytes) return REHYAT_ENOMEM;
  return run_attention(q, k, v, P, static_cast<uint8_t*>(workspace), out, nullptr, nullptr, nullptr, nullptr,
                       nullptr, static_cast<cudaStream_t>(stream));
}

REHYAT_API int rehyat_forward_ws(const void* q, const void* k, const void* v, int B, int H, int F, int S_tok,
                                 int d, int chunk_frames, int overlap_frames, void* out, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  // every pointer is checked before the first stage launches anything
  if (check_qkvo(q, k, v, out)) return REHYAT_EINVAL;
  int st = rehyat_forward_states(k, v, B, H, F, S_tok, d, chunk_frames, overlap_frames, workspace,
                                 workspace_bytes, stream);
  if (st != REHYAT_OK) return st;
  return rehyat_forward_attention(q, k, v, B, H, F, S_tok, d, chunk_frames, overlap_frames, out, workspace,
                                  workspace_bytes, stream);
}

REHYAT_API int rehyat_forward(const void* q, const void* k, const void* v, int B, int H, int F, int S_tok, int d,
                              int chunk_frames, int overlap_frames, void* out, void* stream) {
  FwdPlan P;
  int st = plan_forward(B, H, F, S_tok, d, chunk_frames, overlap_frames, &P);
  if (st != REHYAT_OK) return st;
  if (check_qkvo(q, k, v, out)) return REHYAT_EINVAL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  WsGuard ws(s);
  st = ws.alloc(P.bytes);
  if (st != REHYAT_OK) return st;
  return rehyat_forward_ws(q, k, v, B, H, F, S_tok, d, chunk_frames, overlap_frames, out, ws.p, P.bytes, stream);
}

REHYAT_API int rehyat_forward_ex_workspace_bytes(int B, int H, int F, int S_tok, int d, int chunk_frames,
                                                 int overlap_frames, int sets, size_t* bytes) {
  if (bytes == nullptr) return REHYAT_EINVAL;
  FwdPlan P;
  int st = plan_forward_sets(B, H, F, S_tok, d, chunk_frames, overlap_frames, sets, &P);
  if (st != REHYAT_OK) return st;
  *bytes = P.bytes;
  return REHYAT_OK;
}

REHYAT_API int rehyat_forward_ex(const void* q, const void* k, const void* v, int B, int H, int F, int S_tok, int d,
                                 int chunk_frames, int overlap_frames, int sets, int layout, void* out,
                                 void* workspace, size_t workspace_bytes, void* stream) {
  FwdPlan P;
  int st = plan_forward_sets(B, H, F, S_tok, d, chunk_frames, overlap_frames, sets, &P);
  if (st != REHYAT_OK) return st;
  st = apply_layout(layout, &P);
  if (st != REHYAT_OK) return st;
  if (check_qkvo(q, k, v, out)) return REHYAT_EINVAL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  WsGuard own(s);
  if (workspace == nullptr) {
    st = own.alloc(P.bytes);
    if (st != REHYAT_OK) return st;
    workspace = own.p;
  } else {
    if (reinterpret_cast<uintptr_t>(workspace) % 256 != 0) return REHYAT_EINVAL;
    if (workspace_bytes < P.bytes) return REHYAT_ENOMEM;
  }
  uint8_t* w = static_cast<uint8_t*>(workspace);
  st = run_states(k, v, P, w, nullptr, nullptr, s);
  if (st != REHYAT_OK) return st;
  return run_attention(q, k, v, P, w, out, nullptr, nullptr, nullptr, nullptr, nullptr, s);
}

namespace {
// Device copies of q, k, v, out, then the forward's own scratch.
size_t host_tensor_bytes(const FwdPlan& P) { return align256(static_cast<size_t>(P.BH) * P.N * P.D * 2); }
}  // namespace

REHYAT_API int rehyat_forward_host_workspace_bytes(int B, int H, int F, int S_tok, int d, int chunk_frames,
                                                   int overlap_frames, int sets, size_t* bytes) {
  if (bytes == nullptr) return REHYAT_EINVAL;
  FwdPlan P;
  int st = plan_forward_sets(B, H, F, S_tok, d, chunk_frames, overlap_frames, sets, &P);
  if (st != REHYAT_OK) return st;
  *bytes = 4 * host_tensor_bytes(P) + P.bytes;
  return REHYAT_OK;
}

REHYAT_API int rehyat_forward_host(const void* q_host, const void* k_host, const void* v_host, int B, int H, int F,
                                   int S_tok, int d, int chunk_frames, int overlap_frames, int sets, int layout,
                                   void* out_host, void* workspace, size_t workspace_bytes, void* stream) {
  FwdPlan P;
  int st = plan_forward_sets(B, H, F, S_tok, d, chunk_frames, overlap_frames, sets, &P);
  if (st != REHYAT_OK) return st;
  st = apply_layout(layout, &P);
  if (st != REHYAT_OK) return st;
  if (q_host == nullptr || k_host == nullptr || v_host == nullptr || out_host == nullptr || workspace == nullptr)
    return REHYAT_EINVAL;
  if (reinterpret_cast<uintptr_t>(workspace) % 256 != 0) return REHYAT_EINVAL;
  const size_t tb = host_tensor_bytes(P);
  if (workspace_bytes < 4 * tb + P.bytes) return REHYAT_ENOMEM;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* w = static_cast<uint8_t*>(workspace);
  uint8_t *qd = w, *kd = w + tb, *vd = w + 2 * tb, *od = w + 3 * tb;
  const size_t n = static_cast<size_t>(P.BH) * P.N * P.D * 2;  // bytes of one tensor
  // keys and values first: the states stage needs only them
  if (cudaMemcpyAsync(kd, k_host, n, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(vd, v_host, n, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(qd, q_host, n, cudaMemcpyHostToDevice, s) != cudaSuccess) {
    (void)cudaGetLastError();
    return REHYAT_ECUDA;
  }
  st = run_states(kd, vd, P, w + 4 * tb, nullptr, nullptr, s);
  if (st != REHYAT_OK) return st;
  st = run_attention(qd, kd, vd, P, w + 4 * tb, od, nullptr, nullptr, nullptr, nullptr, nullptr, s);
  if (st != REHYAT_OK) return st;
  if (cudaMemcpyAsync(out_host, od, n, cudaMemcpyDeviceToHost, s) != cudaSuccess) {
    (void)cudaGetLastError();
    return REHYAT_ECUDA;
  }
  return REHYAT_OK;
}

REHYAT_API int rehyat_phi_mlp(const void* x, int B, int H, int N, int d, int layout, const void* W1,
                              const float* b1, const void* W2, const float* b2, void* phi, void* stream) {
  if (B < 1 || H < 1 || N < 1) return REHYAT_EINVAL;
  int st = check_d(d);
  if (st != REHYAT_OK) return st;
  if (static_cast<long long>(B) * H > INT_MAX / 2 || static_cast<long long>(B) * H * N * d > (1LL << 46))
    return REHYAT_EINVAL;
  const long long Nl = N, dl = d, Hl = H;
  long long rs, hs, bs;
  if (layout == REHYAT_LAYOUT_BHND) {
    rs = dl; hs = Nl * dl; bs = Hl * Nl * dl;
  } else if (layout == REHYAT_LAYOUT_BNHD) {
    rs = Hl * dl; hs = dl; bs = Nl * Hl * dl;
  } else {
    return REHYAT_EINVAL;
  }
  const MlpArgs a{x, W1, b1, W2, b2, phi};
  if (check_mlp_args(a)) return REHYAT_EINVAL;
  return run_phi_mlp(&a, 1, B, H, N, d, rs, hs, bs, static_cast<cudaStream_t>(stream));
}

REHYAT_API int rehyat_forward_phi(const void* q, const void* k, const void* v, const void* phi_q, const void* phi_k,
                                  int B, int H, int F, int S_tok, int d, int chunk_frames, int overlap_frames,
                                  int sets, int layout, void* out, void* workspace, size_t workspace_bytes,
                                  void* stream) {
  FwdPlan P;
  int st = plan_forward_sets(B, H, F, S_tok, d, chunk_frames, overlap_frames, sets, &P);
  if (st != REHYAT_OK) return st;
  st = apply_layout(layout, &P);
  if (st != REHYAT_OK) return st;
  if (check_qkvo(q, k, v, out) || check_ptr(phi_q) || check_ptr(phi_k)) return REHYAT_EINVAL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  WsGuard own(s);
  if (workspace == nullptr) {
    st = own.alloc(P.bytes);
    if (st != REHYAT_OK) return st;
    workspace = own.p;
  } else {
    if (reinterpret_cast<uintptr_t>(workspace) % 256 != 0) return REHYAT_EINVAL;
    if (workspace_bytes < P.bytes) return REHYAT_ENOMEM;
  }
  uint8_t* w = static_cast<uint8_t*>(workspace);
  st = run_states(k, v, P, w, nullptr, nullptr, s, phi_k);
  if (st != REHYAT_OK) return st;
  return run_attention(q, k, v, P, w, out, nullptr, nullptr, nullptr, nullptr, nullptr, s, phi_q);
}

namespace {
// Workspace of the learned-map forward: phi(q), phi(k), then the forward's.
size_t mlp_phi_bytes(const FwdPlan& P) { return align256(static_cast<size_t>(P.BH) * P.N * 2 * P.D * 2); }
}  // namespace

REHYAT_API int rehyat_forward_mlp_workspace_bytes(int B, int H, int F, int S_tok, int d, int chunk_frames,
                                                  int overlap_frames, int sets, size_t* bytes) {
  if (bytes == nullptr) return REHYAT_EINVAL;
  FwdPlan P;
  int st = plan_forward_sets(B, H, F, S_tok, d, chunk_frames, overlap_frames, sets, &P);
  if (st != REHYAT_OK) return st;
  *bytes = 2 * mlp_phi_bytes(P) + P.bytes;
  return REHYAT_OK;
}

REHYAT_API int rehyat_forward_mlp(const void* q, const void* k, const void* v, const void* Wq1, const float* bq1,
                                  const void* Wq2, const float* bq2, const void* Wk1, const float* bk1,
                                  const void* Wk2, const float* bk2, int B, int H, int F, int S_tok, int d,
                                  int chunk_frames, int overlap_frames, int sets, int layout, void* out,
                                  void* workspace, size_t workspace_bytes, void* stream) {
  FwdPlan P;
  int st = plan_forward_sets(B, H, F, S_tok, d, chunk_frames, overlap_frames, sets, &P);
  if (st != REHYAT_OK) return st;
  st = apply_layout(layout, &P);
  if (st != REHYAT_OK) return st;
  if (check_qkvo(q, k, v, out)) return REHYAT_EINVAL;
  const void* wts[8] = {Wq1, bq1, Wq2, bq2, Wk1, bk1, Wk2, bk2};
  for (const void* w : wts)
    if (check_ptr(w)) return REHYAT_EINVAL;
  const size_t phi_bytes = mlp_phi_bytes(P);
  const size_t need = 2 * phi_bytes + P.bytes;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  WsGuard own(s);
  if (workspace == nullptr) {
    st = own.alloc(need);
    if (st != REHYAT_OK) return st;
    workspace = own.p;
  } else {
    if (reinterpret_cast<uintptr_t>(workspace) % 256 != 0) return REHYAT_EINVAL;
    if (workspace_bytes < need) return REHYAT_ENOMEM;
  }
  uint8_t* w = static_cast<uint8_t*>(workspace);
  const MlpArgs maps[2] = {{q, Wq1, bq1, Wq2, bq2, w}, {k, Wk1, bk1, Wk2, bk2, w + phi_bytes}};
  st = run_phi_mlp(maps, 2, P.B, P.H, P.N, P.D, P.rs, P.hs, P.bs, s);
  if (st != REHYAT_OK) return st;
  uint8_t* fw = w + 2 * phi_bytes;
  st = run_states(k, v, P, fw, nullptr, nullptr, s, w + phi_bytes);
  if (st != REHYAT_OK) return st;
  return run_attention(q, k, v, P, fw, out, nullptr, nullptr, nullptr, nullptr, nullptr, s, w);
}

REHYAT_API int rehyat_forward_parts(const void* q, const void* k, const void* v, int B, int H, int F, int S_tok,
                                    int d, int chunk_frames, int overlap_frames, float* aS, float* nS, float* aL,
                                    float* nL, float* M, void* stream) {
  FwdPlan P;
  int st = plan_forward(B, H, F, S_tok, d, chunk_frames, overlap_frames, &P);
  if (st != REHYAT_OK) return st;
  if (check_ptr(q) || check_ptr(k) || check_ptr(v) || check_ptr(aS) || check_ptr(aL) || nS == nullptr ||
      nL == nullptr || M == nullptr)
    return REHYAT_EINVAL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  WsGuard ws(s);
  st = ws.alloc(P.bytes);
  if (st != REHYAT_OK) return st;
  uint8_t* w = static_cast<uint8_t*>(ws.p);
  st = run_states(k, v, P, w, nullptr, nullptr, s);
  if (st != REHYAT_OK) return st;
  return run_attention(q, k, v, P, w, nullptr, aS, nS, aL, nL, M, s);
}

REHYAT_API int rehyat_chunk_states(const void* k, const void* v, int B, int H, int F, int S_tok, int d,
                                   int chunk_frames, int overlap_frames, float* S, float* z, void* stream) {
  FwdPlan P;
  int st = plan_forward(B, H, F, S_tok, d, chunk_frames, overlap_frames, &P);
  if (st != REHYAT_OK) return st;
  if (check_ptr(k) || check_ptr(v) || check_ptr(S) || z == nullptr) return REHYAT_EINVAL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  WsGuard ws(s);
  st = ws.alloc(P.off_hi);  // partials only
  if (st != REHYAT_OK) return st;
  return run_states(k, v, P, static_cast<uint8_t*>(ws.p), S, z, s);
}

namespace {
// fp32 forward with optional precomputed features (null: the fixed phi).
int run_forward_f32(const float* q, const float* k, const float* v, const float* phi_q, const float* phi_k, int B,
                    int H, int F, int S_tok, int d, int chunk_frames, int overlap_frames, float* out, void* stream);
}  // namespace

REHYAT_API int rehyat_forward_f32(const float* q, const float* k, const float* v, int B, int H, int F, int S_tok,
                                  int d, int chunk_frames, int overlap_frames, float* out, void* stream) {
  return run_forward_f32(q, k, v, nullptr, nullptr, B, H, F, S_tok, d, chunk_frames, overlap_frames, out, stream);
}

REHYAT_API int rehyat_forward_phi_f32(const float* q, const float* k, const float* v, const float* phi_q,
                                      const float* phi_k, int B, int H, int F, int S_tok, int d, int chunk_frames,
                                      int overlap_frames, float* out, void* stream) {
  if (check_ptr(phi_q) || check_ptr(phi_k)) return REHYAT_EINVAL;
  return run_forward_f32(q, k, v, phi_q, phi_k, B, H, F, S_tok, d, chunk_frames, overlap_frames, out, stream);
}

REHYAT_API int rehyat_phi_mlp_f32(const float* x, int B, int H, int N, int d, const float* W1, const float* b1,
                                  const float* W2, const float* b2, float* phi, void* stream) {
  if (B < 1 || H < 1 || N < 1) return REHYAT_EINVAL;
  int st = check_d(d);
  if (st != REHYAT_OK) return st;
  if (check_ptr(x) || check_ptr(W1) || check_ptr(b1) || check_ptr(W2) || check_ptr(b2) || check_ptr(phi))
    return REHYAT_EINVAL;
  const long long rows = static_cast<long long>(B) * H * N;
  if (rows * d > (1LL << 46)) return REHYAT_EINVAL;
  return cuda_status(launch_phi_mlp_f32(x, rows, N, H, d, W1, b1, W2, b2, phi, static_cast<cudaStream_t>(stream)));
}

namespace {
int run_forward_f32(const float* q, const float* k, const float* v, const float* phi_q, const float* phi_k, int B,
                    int H, int F, int S_tok, int d, int chunk_frames, int overlap_frames, float* out, void* stream) {
  FwdPlan P;
  int st = plan_forward(B, H, F, S_tok, d, chunk_frames, overlap_frames, &P);
  if (st != REHYAT_OK) return st;
  if (P.f32_bytes == 0) return REHYAT_EINVAL;
  if (check_qkvo(q, k, v, out)) return REHYAT_EINVAL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  WsGuard ws(s);
  st = ws.alloc(P.f32_bytes);
  if (st != REHYAT_OK) return st;
  uint8_t* w = static_cast<uint8_t*>(ws.p);
  float* pS = reinterpret_cast<float*>(w + P.f32_off_pS);
  float* pz = reinterpret_cast<float*>(w + P.f32_off_pz);
  float* Sf = reinterpret_cast<float*>(w + P.f32_off_S);
  float* zt = reinterpret_cast<float*>(w + P.f32_off_zt);
  StateF32Params sp{};
  sp.sg = SegGeom{P.N, P.chunk_tok, P.ovl_tok, P.n_seg, 1, 0, 0};
  sp.BH = P.BH;
  sp.D = P.D;
  sp.k = k;
  sp.v = v;
  sp.part_S = pS;
  sp.part_z = pz;
  sp.phi_k = phi_k;
  st = cuda_status(launch_chunk_state_f32(sp, s));
  if (st != REHYAT_OK) return st;
  st = cuda_status(launch_state_scan(pS, pz, P.BH, P.n_seg, 1, P.nc, P.D, nullptr, nullptr, Sf, zt, s));
  if (st != REHYAT_OK) return st;
  AttnF32Params ap{};
  ap.g = ChunkGeom{P.N, P.N, P.chunk_tok, P.ovl_tok, P.nc, 0};
  ap.BH = P.BH;
  ap.D = P.D;
  ap.q = q; ap.k = k; ap.v = v;
  ap.S = Sf;
  ap.S_bh = 2LL * P.D * P.D * P.nc;
  ap.S_t = 2LL * P.D * P.D;
  ap.z = zt;
  ap.z_bh = 2LL * P.D * P.nc;
  ap.z_t = 2LL * P.D;
  ap.out = out;
  ap.phi_q = phi_q;
  return cuda_status(launch_attention_f32(ap, P.nc, s));
}
}  // namespace

// ---------------------------------------------------------------------------
// recurrent form
// ---------------------------------------------------------------------------
REHYAT_API int rehyat_step_workspace_bytes(int B, int H, int S_tok, int d, int q_frames, int ctx_frames,
                                           int evict_frames, size_t* bytes) {
  if (bytes == nullptr) return REHYAT_EINVAL;
  StepPlan P;
  int st = plan_step(B, H, S_tok, d, q_frames, ctx_frames, evict_frames, &P);
  if (st != REHYAT_OK) return st;
  *bytes = P.bytes;
  return REHYAT_OK;
}

namespace {
// One step of the recurrent form: split the carried state into bf16 hi/lo,
// the fused attention of the chunk, then fold the evicted keys into the
// state.  phi_q / phi_k (optional): precomputed features of the chunk's
// queries and of the window's keys ([B, H, Lq, 2d], [B, H, Lk, 2d]).
int run_step(const void* q_c, const void* k_c, const void* v_c, const void* phi_q, const void* phi_k, float* state_S,
             float* state_z, void* out_c, const StepPlan& P, uint8_t* w, cudaStream_t s,
             int layout = REHYAT_LAYOUT_BHND) {
  __nv_bfloat16* hi = reinterpret_cast<__nv_bfloat16*>(w + P.off_hi);
  __nv_bfloat16* lo = reinterpret_cast<__nv_bfloat16*>(w + P.off_lo);
  int st = cuda_status(launch_state_split(state_S, static_cast<long long>(P.BH) * 2 * P.D * P.D, hi, lo, s));
  if (st != REHYAT_OK) return st;
  AttnParams ap;
  std::memset(&ap, 0, sizeof(ap));
  const long long d_ = P.D, H_ = P.H, Nq_ = P.Nq, Nk_ = P.Nk, D2 = 2LL * P.D;
  // element strides of a row, a head and a batch for q / out (rows Nq) and k / v (rows Nk)
  const bool bnhd = layout == REHYAT_LAYOUT_BNHD;
  const long long q_rs = bnhd ? H_ * d_ : d_, q_hs = bnhd ? d_ : Nq_ * d_, q_bs = H_ * Nq_ * d_;
  const long long k_rs = bnhd ? H_ * d_ : d_, k_hs = bnhd ? d_ : Nk_ * d_, k_bs = H_ * Nk_ * d_;
  if (!make_map4(&ap.tm_q, q_c, P.D, P.Nq, P.H, P.B, q_rs, q_hs, q_bs, 128) ||
      !make_map4(&ap.tm_k, k_c, P.D, P.Nk, P.H, P.B, k_rs, k_hs, k_bs, 128) ||
      !make_map4(&ap.tm_v, v_c, P.D, P.Nk, P.H, P.B, k_rs, k_hs, k_bs, 128) ||
      !make_map(&ap.tm_hi, hi, P.D, 2LL * P.D, P.BH, 128) || !make_map(&ap.tm_lo, lo, P.D, 2LL * P.D, P.BH, 128))
    return REHYAT_ECUDA;
  ap.g = ChunkGeom{P.Nq, P.Nk, P.Nq, 0, 1, 1};
  ap.BH = P.BH;
  ap.H = P.H;
  ap.o_sb = q_bs;
  ap.o_sh = q_hs;
  ap.o_sr = q_rs;
  ap.pairs = P.pairs;
  ap.pair_major = 1;
  ap.split_begin = P.split_begin;
  ap.n_split = P.n_split;
  ap.part = reinterpret_cast<float*>(w + P.off_part);
  ap.state_mul = 1;
  ap.scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(P.D));
  ap.z = state_z;
  ap.z_bh = 2LL * P.D;
  ap.z_t = 0;
  ap.out = static_cast<__nv_bfloat16*>(out_c);
  // The attention, the fold of the evicted keys and the state update each
  // follow the previous kernel with a programmatic dependency: the fold
  // (which reads only this chunk's keys and values) fills the SMs the
  // attention's last wave leaves idle; each kernel waits before it touches
  // what an earlier one writes (the attention before its state tiles, the
  // update before everything).
  const int n_ctas = P.n_units + P.n_split;
  if (phi_q != nullptr) {
    ap.phi_q = static_cast<const __nv_bfloat16*>(phi_q);
    st = cuda_status(launch_attention_phi(P.D, ap, n_ctas, s, true));
  } else {
    st = cuda_status(launch_attention(P.D, false, ap, n_ctas, s, true));
  }
  if (st == REHYAT_OK)
    st = cuda_status(launch_split_merge(ap.part, P.n_split, P.split_begin, P.BH, P.H, P.Nq, P.D, ap.out, ap.o_sb,
                                        ap.o_sh, ap.o_sr, s, true));
  if (st != REHYAT_OK || P.evict_tok == 0) return st;
  StateParams sp;
  std::memset(&sp, 0, sizeof(sp));
  if ((phi_k == nullptr && !make_map4(&sp.tm_k, k_c, P.D, P.Nk, P.H, P.B, k_rs, k_hs, k_bs, 64)) ||
      (phi_k != nullptr && !make_map4(&sp.tm_phik, phi_k, D2, P.Nk, P.H, P.B, D2, Nk_ * D2, H_ * Nk_ * D2, 64)) ||
      !make_map4(&sp.tm_v, v_c, P.D, P.Nk, P.H, P.B, k_rs, k_hs, k_bs, 64))
    return REHYAT_ECUDA;
  sp.sg = SegGeom{P.Nk, 0, 0, 1, P.nsplit, 1, P.evict_tok};
  sp.BH = P.BH;
  sp.H = P.H;
  sp.part_S = reinterpret_cast<float*>(w + P.off_pS);
  sp.part_z = reinterpret_cast<float*>(w + P.off_pz);
  st = cuda_status(phi_k != nullptr ? launch_chunk_state_phi(P.D, sp, P.BH * P.nsplit, s, true)
                                    : launch_chunk_state(P.D, sp, P.BH * P.nsplit, s, true));
  if (st != REHYAT_OK) return st;
  return cuda_status(launch_state_accumulate(sp.part_S, sp.part_z, P.BH, P.nsplit, P.D, state_S, state_z, s, true));
}
}  // namespace

REHYAT_API int rehyat_step_ws(const void* q_c, const void* k_c, const void* v_c, float* state_S, float* state_z,
                              void* out_c, int B, int H, int S_tok, int d, int q_frames, int ctx_frames,
                              int evict_frames, void* workspace, size_t workspace_bytes, void* stream) {
  StepPlan P;
  int st = plan_step(B, H, S_tok, d, q_frames, ctx_frames, evict_frames, &P);
  if (st != REHYAT_OK) return st;
  if (check_qkvo(q_c, k_c, v_c, out_c) || check_ptr(state_S) || check_ptr(state_z) || check_ptr(workspace))
    return REHYAT_EINVAL;
  if (reinterpret_cast<uintptr_t>(workspace) % 256 != 0) return REHYAT_EINVAL;
  if (workspace_bytes < P.bytes) return REHYAT_ENOMEM;
  return run_step(q_c, k_c, v_c, nullptr, nullptr, state_S, state_z, out_c, P, static_cast<uint8_t*>(workspace),
                  static_cast<cudaStream_t>(stream));
}

REHYAT_API int rehyat_step_phi(const void* q_c, const void* k_c, const void* v_c, const void* phi_q_c,
                               const void* phi_k_c, float* state_S, float* state_z, void* out_c, int B, int H,
                               int S_tok, int d, int q_frames, int ctx_frames, int evict_frames, void* workspace,
                               size_t workspace_bytes, void* stream) {
  StepPlan P;
  int st = plan_step(B, H, S_tok, d, q_frames, ctx_frames, evict_frames, &P);
  if (st != REHYAT_OK) return st;
  if (check_qkvo(q_c, k_c, v_c, out_c) || check_ptr(state_S) || check_ptr(state_z) || check_ptr(phi_q_c) ||
      check_ptr(phi_k_c))
    return REHYAT_EINVAL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  WsGuard own(s);
  if (workspace == nullptr) {
    st = own.alloc(P.bytes);
    if (st != REHYAT_OK) return st;
    workspace = own.p;
  } else {
    if (reinterpret_cast<uintptr_t>(workspace) % 256 != 0) return REHYAT_EINVAL;
    if (workspace_bytes < P.bytes) return REHYAT_ENOMEM;
  }
  return run_step(q_c, k_c, v_c, phi_q_c, phi_k_c, state_S, state_z, out_c, P, static_cast<uint8_t*>(workspace), s);
}

REHYAT_API int rehyat_step_ex(const void* q_c, const void* k_c, const void* v_c, float* state_S, float* state_z,
                              void* out_c, int B, int H, int S_tok, int d, int q_frames, int ctx_frames,
                              int evict_frames, int layout, void* workspace, size_t workspace_bytes, void* stream) {
  StepPlan P;
  int st = plan_step(B, H, S_tok, d, q_frames, ctx_frames, evict_frames, &P);
  if (st != REHYAT_OK) return st;
  if (layout != REHYAT_LAYOUT_BHND && layout != REHYAT_LAYOUT_BNHD) return REHYAT_EINVAL;
  if (check_qkvo(q_c, k_c, v_c, out_c) || check_ptr(state_S) || check_ptr(state_z)) return REHYAT_EINVAL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  WsGuard own(s);
  if (workspace == nullptr) {
    st = own.alloc(P.bytes);
    if (st != REHYAT_OK) return st;
    workspace = own.p;
  } else {
    if (reinterpret_cast<uintptr_t>(workspace) % 256 != 0) return REHYAT_EINVAL;
    if (workspace_bytes < P.bytes) return REHYAT_ENOMEM;
  }
  return run_step(q_c, k_c, v_c, nullptr, nullptr, state_S, state_z, out_c, P, static_cast<uint8_t*>(workspace), s,
                  layout);
}

REHYAT_API int rehyat_step(const void* q_c, const void* k_c, const void* v_c, float* state_S, float* state_z,
                           void* out_c, int B, int H, int S_tok, int d, int q_frames, int ctx_frames,
                           int evict_frames, void* stream) {
  StepPlan P;
  int st = plan_step(B, H, S_tok, d, q_frames, ctx_frames, evict_frames, &P);
  if (st != REHYAT_OK) return st;
  if (check_qkvo(q_c, k_c, v_c, out_c) || check_ptr(state_S) || check_ptr(state_z)) return REHYAT_EINVAL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  WsGuard ws(s);
  st = ws.alloc(P.bytes);
  if (st != REHYAT_OK) return st;
  return rehyat_step_ws(q_c, k_c, v_c, state_S, state_z, out_c, B, H, S_tok, d, q_frames, ctx_frames,
                        evict_frames, ws.p, P.bytes, stream);
}

REHYAT_API int rehyat_step_f32(const float* q_c, const float* k_c, const float* v_c, float* state_S,
                               float* state_z, float* out_c, int B, int H, int S_tok, int d, int q_frames,
                               int ctx_frames, int evict_frames, void* stream) {
  StepPlan P;
  int st = plan_step(B, H, S_tok, d, q_frames, ctx_frames, evict_frames, &P);
  if (st != REHYAT_OK) return st;
  if (check_qkvo(q_c, k_c, v_c, out_c) || check_ptr(state_S) || check_ptr(state_z)) return REHYAT_EINVAL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  AttnF32Params ap{};
  ap.g = ChunkGeom{P.Nq, P.Nk, P.Nq, 0, 1, 1};
  ap.BH = P.BH;
  ap.D = P.D;
  ap.q = q_c; ap.k = k_c; ap.v = v_c;
  ap.S = state_S;
  ap.S_bh = 2LL * P.D * P.D;
  ap.S_t = 0;
  ap.z = state_z;
  ap.z_bh = 2LL * P.D;
  ap.z_t = 0;
  ap.out = out_c;
  st = cuda_status(launch_attention_f32(ap, 1, s));
  if (st != REHYAT_OK || P.evict_tok == 0) return st;
  WsGuard ws(s);
  st = ws.alloc(P.f32_bytes);
  if (st != REHYAT_OK) return st;
  uint8_t* w = static_cast<uint8_t*>(ws.p);
  StateF32Params sp{};
  sp.sg = SegGeom{P.Nk, 0, 0, 1, 1, 1, P.evict_tok};
  sp.BH = P.BH;
  sp.D = P.D;
  sp.k = k_c;
  sp.v = v_c;
  sp.part_S = reinterpret_cast<float*>(w + P.f32_off_pS);
  sp.part_z = reinterpret_cast<float*>(w + P.f32_off_pz);
  st = cuda_status(launch_chunk_state_f32(sp, s));
  if (st != REHYAT_OK) return st;
  return cuda_status(launch_state_accumulate(sp.part_S, sp.part_z, P.BH, 1, P.D, state_S, state_z, s));
}

// ---------------------------------------------------------------------------
// feature map, status
// ---------------------------------------------------------------------------
REHYAT_API int rehyat_phi(const void* x, int x_dtype, void* y, int y_dtype, int64_t rows, int d, void* stream) {
  if (x == nullptr || y == nullptr || rows < 1 || d < 1) return REHYAT_EINVAL;
  if ((x_dtype != REHYAT_DTYPE_BF16 && x_dtype != REHYAT_DTYPE_F32) ||
      (y_dtype != REHYAT_DTYPE_BF16 && y_dtype != REHYAT_DTYPE_F32))
    return REHYAT_EINVAL;
  if (rows > (1LL << 40) / d) return REHYAT_EINVAL;
  // element accesses: each pointer aligned to its element size
  if (reinterpret_cast<uintptr_t>(x) % (x_dtype == REHYAT_DTYPE_F32 ? 4 : 2) != 0 ||
      reinterpret_cast<uintptr_t>(y) % (y_dtype == REHYAT_DTYPE_F32 ? 4 : 2) != 0)
    return REHYAT_EINVAL;
  return cuda_status(launch_phi(x, x_dtype == REHYAT_DTYPE_F32, y, y_dtype == REHYAT_DTYPE_F32, rows, d,
                                static_cast<cudaStream_t>(stream)));
}

REHYAT_API int rehyat_wait_probe(int* gave_up, void* stream) {
  return cuda_status(launch_wait_probe(gave_up, static_cast<cudaStream_t>(stream)));
}

REHYAT_API int rehyat_device_status(unsigned int* detail) {
  unsigned int v = 0;
  if (cudaDeviceSynchronize() != cudaSuccess) return REHYAT_ECUDA;
  unsigned int v_mlp = 0, v_states = 0;
  if (read_and_clear_device_error(&v) != cudaSuccess) return REHYAT_ECUDA;
  if (read_and_clear_device_error_mlp(&v_mlp) != cudaSuccess) return REHYAT_ECUDA;
  if (read_and_clear_device_error_states(&v_states) != cudaSuccess) return REHYAT_ECUDA;
  v |= v_mlp | v_states;
  if (detail != nullptr) *detail = v;
  return v == 0 ? REHYAT_OK : REHYAT_ETIMEOUT;
}

// ===========================================================================
// Forward without any allocation (scratch in a fixed device array)
// ===========================================================================
// Some callers cannot allocate device memory at call time: a serving process
// that reserves all of the GPU's memory at start-up and forbids later
// allocation (cudaMalloc can synchronise the device and its latency is
// unbounded), or a plugin whose host framework owns the allocator and offers
// no scratch hook.  rehyat_forward_noalloc serves them: its scratch lives in
// the file-scope array below, which every GPU that loads this library holds
// (REHYAT_NOALLOC_SCRATCH_BYTES each) until the process exits.
//
// In host code the name g_noalloc_scratch is only a host-side stand-in for
// the device array, never a device address; the address is looked up with
// cudaGetSymbolAddress with the device current (first on that device's first
// call) and only that address is handed to kernels and to TMA.  Every call
// made outside stream capture looks it up again, so a device reset (which
// reloads the module, possibly at another address) is picked up by the next
// ordinary call; while a stream is being captured the address of the last
// lookup on that device is used.
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[REHYAT_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 128;
std::mutex g_noalloc_mu;
void* g_noalloc_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device.
int noalloc_scratch(cudaStream_t s, void** addr) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return REHYAT_ECUDA;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cap) != cudaSuccess) {
    (void)cudaGetLastError();
    return REHYAT_ECUDA;
  }
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (cap == cudaStreamCaptureStatusNone || g_noalloc_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      (void)cudaGetLastError();
      return REHYAT_ECUDA;
    }
    g_noalloc_addr[dev] = p;
  }
  *addr = g_noalloc_addr[dev];
  return REHYAT_OK;
}

// The forward's scratch layout with a given number of pieces per segment.
size_t layout_with_nsplit(FwdPlan* P, int nsplit) {
  P->nsplit = nsplit;
  const size_t D2 = 2 * static_cast<size_t>(P->D);
  const size_t segs = static_cast<size_t>(P->BH) * P->n_seg * nsplit;
  const size_t chunks = static_cast<size_t>(P->BH) * P->nc;
  size_t off = 0;
  P->off_pS = off; off += align256(segs * D2 * P->D * 4);
  P->off_pz = off; off += align256(segs * D2 * 4);
  P->off_hi = off; off += align256(chunks * D2 * P->D * 2);
  P->off_lo = off; off += align256(chunks * D2 * P->D * 2);
  P->off_zt = off; off += align256(chunks * D2 * 4);
  P->bytes = off > 0 ? off : 256;
  return P->bytes;
}

}  // namespace

REHYAT_API int rehyat_forward_noalloc(const void* q, const void* k, const void* v, int B, int H, int F, int S_tok,
                                      int d, int chunk_frames, int overlap_frames, void* out, void* stream) {
  FwdPlan P;
  int st = plan_forward(B, H, F, S_tok, d, chunk_frames, overlap_frames, &P);
  if (st != REHYAT_OK) return st;
  if (check_qkvo(q, k, v, out)) return REHYAT_EINVAL;
  // Fewer key pieces per segment shrink the partial sums until they fit.
  int nsplit = P.nsplit;
  while (layout_with_nsplit(&P, nsplit) > REHYAT_NOALLOC_SCRATCH_BYTES && nsplit > 1) --nsplit;
  if (P.bytes > REHYAT_NOALLOC_SCRATCH_BYTES) return REHYAT_ENOMEM;  // problem too large for the array
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  void* ws = nullptr;
  st = noalloc_scratch(s, &ws);
  if (st != REHYAT_OK) return st;
  // Every scratch byte this call reads is first written by this call, so
  // nothing is cleared; calls that overlap on the GPU share the array and race.
  uint8_t* w = static_cast<uint8_t*>(ws);
  st = run_states(k, v, P, w, nullptr, nullptr, s);
  if (st != REHYAT_OK) return st;
  return run_attention(q, k, v, P, w, out, nullptr, nullptr, nullptr, nullptr, nullptr, s);
}

#ifdef REHYAT_TRACE
// Trace builds only: where the fused kernel writes its cycle stamps.
REHYAT_API void rehyat_trace_buffer(void* buf) { g_trace = static_cast<unsigned long long*>(buf); }
#endif
