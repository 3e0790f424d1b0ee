// liblinattn.so: the C-ABI host layer (argument checks, kernel choice,
// launch configuration) over the sm_100a kernels.  See include/linattn.h for
// the contract of every entry point.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <atomic>
#include <mutex>
#include <set>
#include <utility>

#include "../../include/linattn.h"
#include "sm100.cuh"
#include "common.cuh"
#include "decode.cuh"
#include "causal_simt.cuh"
#include "causal_tc.cuh"
#include "causal_seg_tc.cuh"
#include "causal_bwd.cuh"
#include "causal_bwd_tc.cuh"
#include "global_simt.cuh"
#include "global_tc.cuh"
#include "performer.cuh"

namespace linattn {
namespace {

constexpr int kVersion = 100;  // 0.1.0

using bf16 = __nv_bfloat16;

bool supported_dim(int d) { return d == 16 || d == 32 || d == 64 || d == 128; }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlaps(const void *a, size_t na, const void *b, size_t nb) {
  if (!a || !b || na == 0 || nb == 0) return false;
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return a0 < b0 + nb && b0 < a0 + na;
}

size_t elem_size(int dtype) { return dtype == LINATTN_F32 ? 4 : 2; }

// Common checks on the dims struct; returns a status code.
int check_dims(const linattn_dims *d, bool use_n) {
  if (!d) return LINATTN_ERR_INVALID;
  if (d->B < 0 || d->H < 0 || (use_n && d->N < 0)) return LINATTN_ERR_INVALID;
  if (d->dtype != LINATTN_BF16 && d->dtype != LINATTN_F32) return LINATTN_ERR_UNSUPPORTED;
  if (d->phi != LINATTN_PHI_ELU1 && d->phi != LINATTN_PHI_IDENTITY) return LINATTN_ERR_UNSUPPORTED;
  if (!supported_dim(d->dk) || !supported_dim(d->dv)) return LINATTN_ERR_UNSUPPORTED;
  const long long n = use_n ? d->N : 1;
  const long long big = static_cast<long long>(d->B) * d->H * n *
                        (d->dk > d->dv ? d->dk : d->dv);
  if (big >= (1ll << 31)) return LINATTN_ERR_UNSUPPORTED;
  if (static_cast<long long>(d->B) * d->H * d->dk * d->dv >= (1ll << 31))
    return LINATTN_ERR_UNSUPPORTED;
  return LINATTN_OK;
}

// q and k hold feature vectors already: the kernels apply no feature map
bool ident(const linattn_dims *d) { return d->phi == LINATTN_PHI_IDENTITY; }

bool bad_eps(float eps) { return !(eps >= 0.f) || !std::isfinite(eps); }

int launch_status() {
  return cudaGetLastError() == cudaSuccess ? LINATTN_OK : LINATTN_ERR_CUDA;
}

// Opt a kernel in to more than 48 KB of dynamic shared memory, once per
// (kernel, device).  Keyed by the kernel's address: instantiations that share
// a signature are still distinct kernels.
bool set_smem_impl(const void *kernel, int bytes) {
  static std::mutex mu;
  static std::set<std::pair<const void *, int>> done;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  std::lock_guard<std::mutex> lock(mu);
  if (done.count({kernel, dev})) return true;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
      cudaSuccess)
    return false;
  done.insert({kernel, dev});
  return true;
}

template <typename F>
bool set_smem(F *kernel, int bytes) {
  return set_smem_impl(reinterpret_cast<const void *>(kernel), bytes);
}

// ------------------------------------------------------------ tensor maps
using EncodeTiled = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                 const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                 const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                 CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled encode_fn() {
  static EncodeTiled fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiled>(p);
  });
  return fn;
}

// [planes, rows, inner] bf16 tensor; boxes of 64 x box_rows x 1 with 128-byte
// swizzle (64 bf16 = 128 bytes per box row).
bool make_map_bf16(CUtensorMap *m, const void *ptr, int inner, int rows, int planes,
                   unsigned box_rows = 128) {
  EncodeTiled enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(rows),
                              static_cast<cuuint64_t>(planes)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(inner) * 2,
                                 static_cast<cuuint64_t>(inner) * rows * 2};
  const cuuint32_t box[3] = {64, box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Kernel family per operation, set by linattn_set_kernel_choice (tests and
// benchmarks compare families on the same call); AUTO unless set.
std::atomic<int> g_choice[4] = {{LINATTN_KERNEL_AUTO}, {LINATTN_KERNEL_AUTO}, {LINATTN_KERNEL_AUTO},
                                {LINATTN_KERNEL_AUTO}};
std::atomic<int> g_forced_segments{0};

int choice(int op) { return g_choice[op].load(std::memory_order_relaxed); }

bool tc_causal_shape(const linattn_dims *d) {
  return d->dtype == LINATTN_BF16 && (d->dk == 128 || d->dk == 64) && (d->dv == 128 || d->dv == 64);
}

// Which causal kernel: bf16 with d_k and d_v in {64, 128} takes the
// segmented tensor-core kernel (one CTA per head and segment, the head's
// whole d_v); the paired kernel (two CTAs per head, d_v split) and the
// CUDA-core kernel are there when chosen explicitly.
enum class CausalPath { kSegTc, kPairedTc, kSimt };
CausalPath causal_path(const linattn_dims *d) {
  const int c = choice(LINATTN_OP_CAUSAL);
  if (c == LINATTN_KERNEL_CUDA_CORES || !tc_causal_shape(d)) return CausalPath::kSimt;
  if (c == LINATTN_KERNEL_TC_PAIRED) return CausalPath::kPairedTc;
  return CausalPath::kSegTc;
}

// ------------------------------------------------------------ launchers
int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

template <int DK, int DV, typename T>
int launch_decode(const linattn_dims *d, const void *q, const void *k, const void *v,
                  const float *lam, float eps, float *S, float *z, void *out,
                  cudaStream_t s) {
  auto *kern = decode_step_kernel<DK, DV, T>;
  const int bytes = static_cast<int>(DecodeLayout<DK, DV, T>::kSmem);
  if (!set_smem(kern, bytes)) return LINATTN_ERR_CUDA;
  const int BH = d->B * d->H;
  const int sms = num_sms();
  if (sms <= 0) return LINATTN_ERR_CUDA;
  const int grid = BH < sms ? BH : sms;
  kern<<<grid, kDecodeThreads, bytes, s>>>(
      static_cast<const T *>(q), static_cast<const T *>(k), static_cast<const T *>(v), lam, eps,
      S, z, static_cast<T *>(out), d->H, BH, ident(d));
  return launch_status();
}

template <int DK, typename T>
int decode_dv(const linattn_dims *d, const void *q, const void *k, const void *v,
              const float *lam, float eps, float *S, float *z, void *out, cudaStream_t s) {
  switch (d->dv) {
    case 16: return launch_decode<DK, 16, T>(d, q, k, v, lam, eps, S, z, out, s);
    case 32: return launch_decode<DK, 32, T>(d, q, k, v, lam, eps, S, z, out, s);
    case 64: return launch_decode<DK, 64, T>(d, q, k, v, lam, eps, S, z, out, s);
    case 128: return launch_decode<DK, 128, T>(d, q, k, v, lam, eps, S, z, out, s);
  }
  return LINATTN_ERR_UNSUPPORTED;
}

template <typename T>
int decode_dispatch(const linattn_dims *d, const void *q, const void *k, const void *v,
                    const float *lam, float eps, float *S, float *z, void *out,
                    cudaStream_t s) {
  switch (d->dk) {
    case 16: return decode_dv<16, T>(d, q, k, v, lam, eps, S, z, out, s);
    case 32: return decode_dv<32, T>(d, q, k, v, lam, eps, S, z, out, s);
    case 64: return decode_dv<64, T>(d, q, k, v, lam, eps, S, z, out, s);
    case 128: return decode_dv<128, T>(d, q, k, v, lam, eps, S, z, out, s);
  }
  return LINATTN_ERR_UNSUPPORTED;
}

// Segment-parallel plan for the CUDA-core causal kernel: G segments of len
// tokens when (b, h, dv-slice) alone would leave most SMs idle; ws is the
// workspace (G = 1: none, single pass).
struct Segments {
  int G = 1, len = 0;
  float *ws = nullptr;
};
constexpr int kMaxSegments = 64;
// time per token of the tensor-core state pass relative to the forward
// (measured on the causal_decay_d128 workload); sets the split of two segments
constexpr double kStatePassCost = 0.4;

int simt_dv_slice(int dv) { return dv <= 16 ? 16 : 32; }

Segments plan_segments(const linattn_dims *d) {
  Segments sg;
  sg.len = d->N;
  if (causal_path(d) != CausalPath::kSimt || d->N < 256) return sg;
  const long ctas = static_cast<long>(d->B) * d->H * (d->dv / simt_dv_slice(d->dv));
  const int sms = num_sms();
  if (sms <= 0 || ctas == 0 || ctas >= sms) return sg;
  long G = (2L * sms + ctas - 1) / ctas;   // about two waves of CTAs
  G = std::min<long>(G, d->N / 128);       // segments of at least 128 tokens
  G = std::min<long>(G, kMaxSegments);
  if (G < 2) return sg;
  const int len = static_cast<int>(((d->N + G - 1) / G + 31) / 32 * 32);
  sg.G = (d->N + len - 1) / len;
  sg.len = len;
  if (sg.G < 2) sg = Segments{1, d->N, nullptr};
  return sg;
}

size_t segment_bytes(const linattn_dims *d, const Segments &sg) {
  if (sg.G < 2) return 0;
  return static_cast<size_t>(d->B) * d->H * sg.G * (static_cast<size_t>(d->dk) * d->dv + d->dk) * 4;
}

template <int DK, int DVS, typename T>
int launch_causal_simt(const linattn_dims *d, const void *q, const void *k, const void *v,
                       const float *lam, float eps, const float *S_init, const float *z_init,
                       void *out, float *S_final, float *z_final, const Segments &sg,
                       cudaStream_t s) {
  auto *kern = causal_simt_kernel<DK, DVS, T>;
  const int bytes = causal_simt_smem_floats<DK, DVS>() * 4;
  if (!set_smem(kern, bytes)) return LINATTN_ERR_CUDA;
  const int ctas = d->B * d->H * (d->dv / DVS);
  float *wsS = sg.ws, *wsz = sg.ws ? sg.ws + static_cast<long>(d->B) * d->H * sg.G * d->dk * d->dv
                                   : nullptr;
  if (sg.G > 1) {
    // (1) each segment's own final state from zero, (2) the starting states
    causal_seg_state_kernel<DK, DVS, T><<<dim3(ctas, sg.G - 1), 256, 0, s>>>(
        static_cast<const T *>(k), static_cast<const T *>(v), lam, wsS, wsz, d->H, d->N, d->dv,
        sg.len, sg.G, ident(d));
    if (cudaGetLastError() != cudaSuccess) return LINATTN_ERR_CUDA;
    const int eblocks = (d->dk * d->dv + d->dk + 255) / 256;
    causal_seg_combine_kernel<<<dim3(d->B * d->H, eblocks), 256, 0, s>>>(
        lam, S_init, z_init, wsS, wsz, d->H, d->dk, d->dv, d->N, sg.len, sg.G, false);
    if (cudaGetLastError() != cudaSuccess) return LINATTN_ERR_CUDA;
  }
  kern<<<dim3(ctas, sg.G), 256, bytes, s>>>(
      static_cast<const T *>(q), static_cast<const T *>(k), static_cast<const T *>(v), lam, eps,
      S_init, z_init, static_cast<T *>(out), S_final, z_final, d->H, d->N, d->dv, sg.len,
      sg.G > 1 ? wsS : nullptr, sg.G > 1 ? wsz : nullptr, ident(d));
  return launch_status();
}

template <int DK, typename T>
int causal_simt_dv(const linattn_dims *d, const void *q, const void *k, const void *v,
                   const float *lam, float eps, const float *S_init, const float *z_init,
                   void *out, float *S_final, float *z_final, const Segments &sg,
                   cudaStream_t s) {
  if (d->dv == 16)
    return launch_causal_simt<DK, 16, T>(d, q, k, v, lam, eps, S_init, z_init, out, S_final,
                                         z_final, sg, s);
  return launch_causal_simt<DK, 32, T>(d, q, k, v, lam, eps, S_init, z_init, out, S_final,
                                       z_final, sg, s);
}

template <typename T>
int causal_simt_dispatch(const linattn_dims *d, const void *q, const void *k, const void *v,
                         const float *lam, float eps, const float *S_init, const float *z_init,
                         void *out, float *S_final, float *z_final, const Segments &sg,
                         cudaStream_t s) {
  switch (d->dk) {
    case 16: return causal_simt_dv<16, T>(d, q, k, v, lam, eps, S_init, z_init, out, S_final, z_final, sg, s);
    case 32: return causal_simt_dv<32, T>(d, q, k, v, lam, eps, S_init, z_init, out, S_final, z_final, sg, s);
    case 64: return causal_simt_dv<64, T>(d, q, k, v, lam, eps, S_init, z_init, out, S_final, z_final, sg, s);
    case 128: return causal_simt_dv<128, T>(d, q, k, v, lam, eps, S_init, z_init, out, S_final, z_final, sg, s);
  }
  return LINATTN_ERR_UNSUPPORTED;
}

// Segment plan of the tensor-core causal kernel: G segments of seg_len
// tokens (whole chunks) when one CTA per head would leave most SMs idle.
struct TcSegments {
  int G = 1, len = 0;
};

// Launch configuration with programmatic stream serialization: the grid may
// begin before the previous grid of the stream has finished, and orders
// itself after it with griddepcontrol.wait where it reads that grid's output.
struct ProgrammaticLaunch {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  ProgrammaticLaunch(int grid, int block, size_t smem, cudaStream_t s) {
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
};

TcSegments plan_tc_segments(const linattn_dims *d) {
  TcSegments sg;
  sg.len = d->N;
  const long BH = static_cast<long>(d->B) * d->H;
  const int nch = (d->N + stc::C - 1) / stc::C;
  const int sms = num_sms();
  if (BH <= 0 || nch < 2 || sms <= 0) return sg;
  long gmax = g_forced_segments.load(std::memory_order_relaxed);
  if (gmax <= 0) gmax = sms / BH;   // about one CTA per SM
  gmax = std::min<long>(gmax, std::min(nch, kMaxSegments));
  if (gmax < 2) return sg;
  int len_ch;
  if (gmax == 2) {
    // Two segments: the first runs beside the state pass over itself, the
    // second after it, so the first is longer by the state pass's share:
    // len0 (1 - a) = len1 with a the state pass's cost per token relative
    // to the forward's.
    len_ch = static_cast<int>(std::ceil(nch / (2.0 - kStatePassCost)));
  } else {
    len_ch = (nch + static_cast<int>(gmax) - 1) / static_cast<int>(gmax);
  }
  sg.G = (nch + len_ch - 1) / len_ch;
  sg.len = len_ch * stc::C;
  if (sg.G < 2) sg = TcSegments{1, d->N};
  return sg;
}

size_t tc_segment_bytes(const linattn_dims *d, const TcSegments &sg) {
  if (sg.G < 2) return 0;
  return static_cast<size_t>(d->B) * d->H * sg.G * (static_cast<size_t>(d->dk) * d->dv + d->dk) * 4;
}

template <int DKP, int DVP>
int launch_causal_seg_tc_t(const linattn_dims *d, const CUtensorMap &mq, const CUtensorMap &mk,
                           const CUtensorMap &mv, const float *lam, float eps,
                           const float *S_init, const float *z_init, void *out, float *S_final,
                           float *z_final, const TcSegments &sg, float *ws, cudaStream_t s) {
  auto *kern = stc::causal_seg_tc_kernel<DKP, DVP>;
  if (!set_smem(kern, static_cast<int>(stc::kSmemBytes))) return LINATTN_ERR_CUDA;
  const int BH = d->B * d->H;
  float *wsS = nullptr, *wsz = nullptr;
  if (sg.G > 1) {
    wsS = ws;
    wsz = ws + static_cast<long>(BH) * sg.G * d->dk * d->dv;
    // each of the first G - 1 segments' own final state from zero; the
    // forward sums them into its starting states
    auto *sk = stc::causal_seg_state_tc_kernel<DKP, DVP>;
    if (!set_smem(sk, static_cast<int>(stc::sp::kSmemBytes))) return LINATTN_ERR_CUDA;
    sk<<<BH * (sg.G - 1), stc::sp::NT, stc::sp::kSmemBytes, s>>>(
        mk, mv, lam, wsS, wsz, d->H, d->N, sg.len, sg.G - 1, sg.G, ident(d));
    if (cudaGetLastError() != cudaSuccess) return LINATTN_ERR_CUDA;
    // the forward as the state pass's dependent: its first segment's CTAs
    // run beside the state pass, the others wait for it (griddepcontrol)
    ProgrammaticLaunch pl(BH * sg.G, stc::NT, stc::kSmemBytes, s);
    if (cudaLaunchKernelEx(&pl.cfg, kern, mq, mk, mv, lam, eps, S_init, z_init,
                           static_cast<const float *>(wsS), static_cast<const float *>(wsz),
                           static_cast<bf16 *>(out), S_final, z_final, d->H, d->N, sg.len, sg.G,
                           ident(d)) != cudaSuccess)
      return LINATTN_ERR_CUDA;
    return launch_status();
  }
  kern<<<BH, stc::NT, stc::kSmemBytes, s>>>(
      mq, mk, mv, lam, eps, S_init, z_init, nullptr, nullptr, static_cast<bf16 *>(out), S_final,
      z_final, d->H, d->N, sg.len, 1, ident(d));
  return launch_status();
}

int launch_causal_seg_tc(const linattn_dims *d, const void *q, const void *k, const void *v,
                         const float *lam, float eps, const float *S_init, const float *z_init,
                         void *out, float *S_final, float *z_final, const TcSegments &sg,
                         float *ws, cudaStream_t s) {
  const int BH = d->B * d->H;
  CUtensorMap mq, mk, mv;
  if (!make_map_bf16(&mq, q, d->dk, d->N, BH) || !make_map_bf16(&mk, k, d->dk, d->N, BH) ||
      !make_map_bf16(&mv, v, d->dv, d->N, BH))
    return LINATTN_ERR_CUDA;
  if (d->dk == 128)
    return d->dv == 128 ? launch_causal_seg_tc_t<2, 2>(d, mq, mk, mv, lam, eps, S_init, z_init, out,
                                                       S_final, z_final, sg, ws, s)
                        : launch_causal_seg_tc_t<2, 1>(d, mq, mk, mv, lam, eps, S_init, z_init, out,
                                                       S_final, z_final, sg, ws, s);
  return d->dv == 128 ? launch_causal_seg_tc_t<1, 2>(d, mq, mk, mv, lam, eps, S_init, z_init, out,
                                                     S_final, z_final, sg, ws, s)
                      : launch_causal_seg_tc_t<1, 1>(d, mq, mk, mv, lam, eps, S_init, z_init, out,
                                                     S_final, z_final, sg, ws, s);
}

int launch_causal_tc(const linattn_dims *d, const void *q, const void *k, const void *v,
                     const float *lam, float eps, const float *S_init, const float *z_init,
                     void *out, float *S_final, float *z_final, cudaStream_t s) {
  const int BH = d->B * d->H;
  // dv = 128: the two column halves of a head run as a 2-CTA cluster that
  // shares the feature map (each CTA loads 64 rows of every q/k tile)
  const bool paired = d->dv == 2 * tc::DVS;
  const unsigned qk_rows = paired ? 64u : 128u;
  CUtensorMap mq, mk, mv;
  if (!make_map_bf16(&mq, q, d->dk, d->N, BH, qk_rows) ||
      !make_map_bf16(&mk, k, d->dk, d->N, BH, qk_rows) || !make_map_bf16(&mv, v, d->dv, d->N, BH))
    return LINATTN_ERR_CUDA;
  const bool half = d->dk == 64;   // d_k = 64: the kernel's second d_k panel stays zero
  auto *kern = paired ? (half ? tc::causal_tc_kernel<true, true> : tc::causal_tc_kernel<true, false>)
                      : (half ? tc::causal_tc_kernel<false, true> : tc::causal_tc_kernel<false, false>);
  if (!set_smem(kern, static_cast<int>(tc::kSmemBytes))) return LINATTN_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(BH * (d->dv / tc::DVS));
  cfg.blockDim = dim3(tc::NT);
  cfg.dynamicSmemBytes = tc::kSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = paired ? 2 : 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, mq, mk, mv, lam, eps, S_init, z_init,
                         static_cast<bf16 *>(out), S_final, z_final, d->H, d->N, d->dv,
                         ident(d)) != cudaSuccess)
    return LINATTN_ERR_CUDA;
  return launch_status();
}

template <int DK, int DV, typename T>
int launch_global_simt(const linattn_dims *d, int Nk, const void *q, const void *k,
                       const void *v, const uint8_t *kpm, float eps, void *out, float *KV,
                       float *ksum, cudaStream_t s) {
  // KV, ksum over the Nk keys (none: they stay zero), then y for the d->N queries
  const int BH = d->B * d->H;
  if (Nk > 0) {
    dim3 g1(BH, (Nk + kGlobalSplit - 1) / kGlobalSplit);
    global_kv_simt_kernel<DK, DV, T><<<g1, 256, 0, s>>>(
        static_cast<const T *>(k), static_cast<const T *>(v), kpm, KV, ksum, Nk, d->H, ident(d));
    if (cudaGetLastError() != cudaSuccess) return LINATTN_ERR_CUDA;
  }
  if (d->N > 0) {
    auto *kern = global_out_simt_kernel<DK, DV, T>;
    const int bytes = (DK * DV + DK + kGlobalTile * (DK + 1) + kGlobalTile) * 4;
    if (!set_smem(kern, bytes)) return LINATTN_ERR_CUDA;
    dim3 g2(BH, (d->N + kGlobalTile - 1) / kGlobalTile);
    kern<<<g2, 256, bytes, s>>>(static_cast<const T *>(q), KV, ksum, eps,
                                static_cast<T *>(out), d->N, ident(d));
  }
  return launch_status();
}

// Tensor-core global path: bf16, d_k = d_v = 64, an even number of heads
// (heads are paired in the KV kernel).  LINATTN_KERNEL_CUDA_CORES chosen for
// the global operation forces the CUDA-core kernels.
bool use_tc_global(const linattn_dims *d) {
  if (choice(LINATTN_OP_GLOBAL) == LINATTN_KERNEL_CUDA_CORES) return false;
  return d->dtype == LINATTN_BF16 && d->dk == gtc::D && d->dv == gtc::D && d->H % 2 == 0;
}

// KV and ksum to zero in one launch
int zero_kv(float *KV, size_t nS, float *ksum, size_t nz, cudaStream_t s) {
  const long n4 = static_cast<long>((nS + nz) / 16);
  const int sms = num_sms();
  const long blocks = std::min<long>((n4 + 255) / 256, 4L * (sms > 0 ? sms : 148));
  if (blocks <= 0) return LINATTN_OK;
  gtc::zero2_kernel<<<static_cast<int>(blocks), 256, 0, s>>>(
      reinterpret_cast<float4 *>(KV), static_cast<long>(nS / 16), reinterpret_cast<float4 *>(ksum),
      static_cast<long>(nz / 16));
  return cudaGetLastError() == cudaSuccess ? LINATTN_OK : LINATTN_ERR_CUDA;
}

int launch_global_tc(const linattn_dims *d, int Nk, const void *q, const void *k,
                     const void *v, const uint8_t *kpm, float eps, void *out, float *KV,
                     float *ksum, cudaStream_t s) {
  // KV, ksum over the Nk keys (none: they stay zero), then y for the d->N queries
  const int BH = d->B * d->H;
  const int sms = num_sms();
  if (sms <= 0) return LINATTN_ERR_CUDA;
  // both kernels run two CTAs per SM: the largest shared-memory carveout
  if (!set_smem(gtc::global_kv_tc_kernel, static_cast<int>(gtc::kv::kSmemBytes)) ||
      !set_smem(gtc::global_out_tc_kernel, static_cast<int>(gtc::out::kSmemBytes)) ||
      cudaFuncSetAttribute(gtc::global_out_tc_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                           cudaSharedmemCarveoutMaxShared) != cudaSuccess ||
      cudaFuncSetAttribute(gtc::global_kv_tc_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                           cudaSharedmemCarveoutMaxShared) != cudaSuccess)
    return LINATTN_ERR_CUDA;
  if (Nk > 0) {
    CUtensorMap mk, mv;
    // 64-token boxes: the KV kernel's units are 64 tokens of a head pair
    if (!make_map_bf16(&mk, k, d->dk, Nk, BH, gtc::kv::CK) ||
        !make_map_bf16(&mv, v, d->dv, Nk, BH, gtc::kv::CK))
      return LINATTN_ERR_CUDA;
    const long u1 = static_cast<long>(BH / 2) * ((Nk + gtc::kv::CK - 1) / gtc::kv::CK);
    // programmatic dependent launch: the KV grid may start while KV / ksum are
    // being zeroed; it waits for that grid only before its first flush.  Two
    // persistent CTAs per SM.
    const int cap1 = gtc::kv::kCtasPerSm * sms;
    const ProgrammaticLaunch pl(static_cast<int>(u1 < cap1 ? u1 : cap1), gtc::kv::NT,
                                gtc::kv::kSmemBytes, s);
    if (cudaLaunchKernelEx(&pl.cfg, gtc::global_kv_tc_kernel, mk, mv, kpm, KV, ksum, BH / 2, Nk,
                           d->H, ident(d)) != cudaSuccess)
      return LINATTN_ERR_CUDA;
  }
  if (d->N > 0) {
    CUtensorMap mq, my;
    if (!make_map_bf16(&mq, q, d->dk, d->N, BH) || !make_map_bf16(&my, out, d->dv, d->N, BH))
      return LINATTN_ERR_CUDA;
    const long u2 = static_cast<long>(BH) * ((d->N + gtc::C - 1) / gtc::C);
    // the output grid loads q and applies phi while the KV grid drains; it
    // waits for that grid only before reading KV and ksum
    // two persistent CTAs per SM (64 registers, 115 KB of shared memory each)
    const int cap2 = gtc::out::kCtasPerSm * sms;
    const ProgrammaticLaunch pl(static_cast<int>(u2 < cap2 ? u2 : cap2), gtc::out::NT,
                                gtc::out::kSmemBytes, s);
    if (cudaLaunchKernelEx(&pl.cfg, gtc::global_out_tc_kernel, mq, my,
                           static_cast<const float *>(KV), static_cast<const float *>(ksum), eps,
                           BH, d->N, ident(d)) != cudaSuccess)
      return LINATTN_ERR_CUDA;
  }
  return launch_status();
}

template <int DK, typename T>
int global_dv(const linattn_dims *d, int Nk, const void *q, const void *k, const void *v,
              const uint8_t *kpm, float eps, void *out, float *KV, float *ksum, cudaStream_t s) {
  switch (d->dv) {
    case 16: return launch_global_simt<DK, 16, T>(d, Nk, q, k, v, kpm, eps, out, KV, ksum, s);
    case 32: return launch_global_simt<DK, 32, T>(d, Nk, q, k, v, kpm, eps, out, KV, ksum, s);
    case 64: return launch_global_simt<DK, 64, T>(d, Nk, q, k, v, kpm, eps, out, KV, ksum, s);
    case 128: return launch_global_simt<DK, 128, T>(d, Nk, q, k, v, kpm, eps, out, KV, ksum, s);
  }
  return LINATTN_ERR_UNSUPPORTED;
}

template <typename T>
int global_dispatch(const linattn_dims *d, int Nk, const void *q, const void *k, const void *v,
                    const uint8_t *kpm, float eps, void *out, float *KV, float *ksum,
                    cudaStream_t s) {
  switch (d->dk) {
    case 16: return global_dv<16, T>(d, Nk, q, k, v, kpm, eps, out, KV, ksum, s);
    case 32: return global_dv<32, T>(d, Nk, q, k, v, kpm, eps, out, KV, ksum, s);
    case 64: return global_dv<64, T>(d, Nk, q, k, v, kpm, eps, out, KV, ksum, s);
    case 128: return global_dv<128, T>(d, Nk, q, k, v, kpm, eps, out, KV, ksum, s);
  }
  return LINATTN_ERR_UNSUPPORTED;
}

template <int DK, int DV, typename T>
int launch_causal_bwd(const linattn_dims *d, const void *q, const void *k, const void *v,
                      const float *lam, float eps, const void *dy, void *dq, void *dk, void *dv,
                      float *dlam, cudaStream_t s) {
  auto *kern = causal_bwd_kernel<DK, DV, T>;
  // the attribute covers the larger layout (with dlambda) once per kernel and device
  if (!set_smem(kern, causal_bwd_smem_floats<DK, DV>(true) * 4)) return LINATTN_ERR_CUDA;
  const int bytes = causal_bwd_smem_floats<DK, DV>(dlam != nullptr) * 4;
  kern<<<d->B * d->H, kBwdThreads, bytes, s>>>(
      static_cast<const T *>(q), static_cast<const T *>(k), static_cast<const T *>(v),
      static_cast<const T *>(dy), lam, eps, static_cast<T *>(dq), static_cast<T *>(dk),
      static_cast<T *>(dv), dlam, d->H, d->N, ident(d));
  return launch_status();
}

template <int DK, typename T>
int causal_bwd_dv(const linattn_dims *d, const void *q, const void *k, const void *v,
                  const float *lam, float eps, const void *dy, void *dq, void *dk, void *dv,
                  float *dlam, cudaStream_t s) {
  switch (d->dv) {
    case 16: return launch_causal_bwd<DK, 16, T>(d, q, k, v, lam, eps, dy, dq, dk, dv, dlam, s);
    case 32: return launch_causal_bwd<DK, 32, T>(d, q, k, v, lam, eps, dy, dq, dk, dv, dlam, s);
    case 64: return launch_causal_bwd<DK, 64, T>(d, q, k, v, lam, eps, dy, dq, dk, dv, dlam, s);
    case 128: return launch_causal_bwd<DK, 128, T>(d, q, k, v, lam, eps, dy, dq, dk, dv, dlam, s);
  }
  return LINATTN_ERR_UNSUPPORTED;
}

// The tensor-core backward: bf16, d_k = d_v = 128.  Pass F (dq, and den,
// dden per token into the stash), pass L (dlambda's carried-derivative part,
// only when dlambda is wanted), pass R (dk, dv).  The stash is a stream-ordered
// allocation of 8 bytes per token, so R (which writes dk) runs beside L as its
// programmatic dependent; without it the stash lives in the dk rows and R
// follows L.
bool use_tc_bwd(const linattn_dims *d) {
  return choice(LINATTN_OP_BACKWARD) != LINATTN_KERNEL_CUDA_CORES && d->dtype == LINATTN_BF16 &&
         d->dk == 128 && d->dv == 128;
}

template <typename... KArgs, typename... Args>
int launch_pdl(void (*kern)(KArgs...), int grid, int block, size_t smem, cudaStream_t s,
               bool programmatic, Args... args) {
  ProgrammaticLaunch pl(grid, block, smem, s);
  if (!programmatic) pl.cfg.numAttrs = 0;
  return cudaLaunchKernelEx(&pl.cfg, kern, args...) == cudaSuccess ? LINATTN_OK
                                                                   : LINATTN_ERR_CUDA;
}

// Split point of pass F (0: one CTA per head), see launch_bwd_tc.
int bwd_split(const linattn_dims *d) {
  const int BH = d->B * d->H;
  const int nch = (d->N + btc::C - 1) / btc::C;
  const int sms = num_sms();
  const int H0 = (nch >= 2 && sms > 0 && BH < sms) ? (nch * 100 + 169) / 170 : 0;
  return H0 >= nch ? 0 : H0;
}

// Workspace of the tensor-core backward: the split-point states of passes F
// and R (when they are split) and the per-token den, dden stash.
size_t bwd_tc_bytes(const linattn_dims *d, int H0) {
  const size_t BH = static_cast<size_t>(d->B) * d->H;
  return (H0 ? 2 * BH * btc::kMidFloats * sizeof(float) : 0) +
         BH * static_cast<size_t>(d->N) * 2 * sizeof(float);
}

// user_ws: the caller's workspace, used when it holds the split form or at
// least the stash; otherwise, with may_alloc, one is allocated on the stream;
// with neither, the stash lives in the dk rows and the passes run in order,
// unsplit.
int launch_bwd_tc(const linattn_dims *d, const void *q, const void *k, const void *v,
                  const float *lam, float eps, const void *dy, void *dq, void *dk, void *dv,
                  float *dlam, void *user_ws, size_t user_bytes, bool may_alloc,
                  cudaStream_t s) {
  const int BH = d->B * d->H;
  CUtensorMap mq, mk, mv, mg;
  if (!make_map_bf16(&mq, q, 128, d->N, BH) || !make_map_bf16(&mk, k, 128, d->N, BH) ||
      !make_map_bf16(&mv, v, 128, d->N, BH) || !make_map_bf16(&mg, dy, 128, d->N, BH))
    return LINATTN_ERR_CUDA;
  if (!set_smem(btc::bwd_tc_f_kernel, static_cast<int>(btc::pf::kSmemBytes)) ||
      !set_smem(btc::bwd_tc_l_kernel, static_cast<int>(btc::pl::kSmemBytes)) ||
      !set_smem(btc::bwd_tc_r_kernel, static_cast<int>(btc::pr::kSmemBytes)) ||
      !set_smem(btc::bwd_tc_s_kernel, static_cast<int>(btc::ps::kSmemBytes)) ||
      !set_smem(btc::bwd_tc_t_kernel, static_cast<int>(btc::pt::kSmemBytes)))
    return LINATTN_ERR_CUDA;
  auto *bq = static_cast<bf16 *>(dq);
  auto *bk = static_cast<bf16 *>(dk);
  auto *bv = static_cast<bf16 *>(dv);
  const bool id = ident(d);
  // Pass F in two halves per head when the heads alone leave SMs idle: the
  // first half from the start, the second from the state at token H0 C
  // (written by the state pass, which runs beside the first halves).  The
  // split point balances the first half against the state pass plus the
  // second half: with the state pass at a fraction a of pass F's time per
  // chunk, H0 = nch / (2 - a); a is ~0.3 (nch / 1.7 timed best against
  // nch / 1.8 at the full-size workload).
  int H0 = bwd_split(d);
  char *ws = nullptr;
  bool owned = false;
  if (user_ws && user_bytes >= bwd_tc_bytes(d, H0)) {
    ws = static_cast<char *>(user_ws);
  } else if (user_ws && user_bytes >= bwd_tc_bytes(d, 0)) {
    ws = static_cast<char *>(user_ws);
    H0 = 0;
  } else if (may_alloc) {
    if (cudaMallocAsync(reinterpret_cast<void **>(&ws), bwd_tc_bytes(d, H0), s) == cudaSuccess) {
      owned = true;
    } else {
      cudaGetLastError();
      ws = nullptr;
    }
  }
  if (!ws) H0 = 0;   // the stash in the dk rows, unsplit
  // pass R splits at H1 = nch - H0 when no dlambda is asked for: its later
  // half (from the end, walked first with no carried adjoint) matches F's
  // first, and the reverse state pass over that half supplies the earlier
  // half's starting adjoint.  With dlambda, R stays one CTA per head beside
  // the dlambda pass: the 64 + 128 + 64 CTAs of L, split R and the reverse
  // state pass leave a tail wave on 148 SMs (3.1 ms against 2.7).
  const int nch = (d->N + btc::C - 1) / btc::C;
  const int H1 = (H0 && !dlam) ? nch - H0 : 0;
  const size_t mid_bytes = bwd_tc_bytes(d, H0) - bwd_tc_bytes(d, 0);
  float *mid = ws ? reinterpret_cast<float *>(ws) : nullptr;
  float *rmid = H0 ? mid + static_cast<size_t>(BH) * btc::kMidFloats : nullptr;
  float *stash = ws ? reinterpret_cast<float *>(ws + mid_bytes) : reinterpret_cast<float *>(dk);
  const long stride = ws ? 2 : btc::D / 2;
  int rc = LINATTN_OK;
  if (H0)
    rc = launch_pdl(btc::bwd_tc_s_kernel, BH, btc::ps::kNT, btc::ps::kSmemBytes, s, false, mk, mv, lam,
                    mid, d->H, d->N, H0, id);
  if (rc == LINATTN_OK)
    rc = launch_pdl(btc::bwd_tc_f_kernel, H0 ? 2 * BH : BH, btc::pf::kNT, btc::pf::kSmemBytes, s,
                    H0 != 0, mq, mk, mv, mg, lam, eps, bq, stash, stride, dlam,
                    static_cast<const float *>(mid), H0, d->H, d->N, id);
  if (rc == LINATTN_OK && dlam)
    rc = launch_pdl(btc::bwd_tc_l_kernel, BH, btc::pl::kNT, btc::pl::kSmemBytes, s, false, mq, mk, mv,
                    mg, lam, static_cast<const float *>(stash), stride, dlam, d->H, d->N, id);
  // R (and the reverse state pass before it) read nothing that L writes: with
  // the stash out of the dk rows they start beside L as programmatic dependents
  const bool beside_l = ws != nullptr && dlam != nullptr;
  if (rc == LINATTN_OK && H1)
    rc = launch_pdl(btc::bwd_tc_t_kernel, BH, btc::pt::kNT, btc::pt::kSmemBytes, s, beside_l, mq, mg,
                    lam, static_cast<const float *>(stash), stride, rmid, d->H, d->N, H1, id);
  if (rc == LINATTN_OK)
    rc = launch_pdl(btc::bwd_tc_r_kernel, H1 ? 2 * BH : BH, btc::pr::kNT, btc::pr::kSmemBytes, s,
                    beside_l || H1 != 0, mq, mk, mv, mg, lam, static_cast<const float *>(stash),
                    stride, bk, bv, static_cast<const float *>(rmid), H1, d->H, d->N, id);
  if (owned && cudaFreeAsync(ws, s) != cudaSuccess && rc == LINATTN_OK) rc = LINATTN_ERR_CUDA;
  return rc;
}

template <typename T>
int causal_bwd_dispatch(const linattn_dims *d, const void *q, const void *k, const void *v,
                        const float *lam, float eps, const void *dy, void *dq, void *dk, void *dv,
                        float *dlam, cudaStream_t s) {
  switch (d->dk) {
    case 16: return causal_bwd_dv<16, T>(d, q, k, v, lam, eps, dy, dq, dk, dv, dlam, s);
    case 32: return causal_bwd_dv<32, T>(d, q, k, v, lam, eps, dy, dq, dk, dv, dlam, s);
    case 64: return causal_bwd_dv<64, T>(d, q, k, v, lam, eps, dy, dq, dk, dv, dlam, s);
    case 128: return causal_bwd_dv<128, T>(d, q, k, v, lam, eps, dy, dq, dk, dv, dlam, s);
  }
  return LINATTN_ERR_UNSUPPORTED;
}

}  // namespace
}  // namespace linattn

using namespace linattn;

namespace linattn {
namespace {

// Both causal entry points: validation, then the tensor-core kernel (bf16,
// d_k = 128, dv a multiple of 64) or the CUDA-core kernel.
int fwd_causal_impl(const linattn_dims *d, const void *q, const void *k, const void *v,
                    const float *lambda, float eps, const float *S_init, const float *z_init,
                    void *out, float *S_final, float *z_final, void *ws, size_t ws_bytes,
                    cudaStream_t s) {
  int rc = check_dims(d, true);
  if (rc != LINATTN_OK) return rc;
  if (bad_eps(eps)) return LINATTN_ERR_INVALID;
  const size_t BH = static_cast<size_t>(d->B) * d->H;
  if (BH == 0) return LINATTN_OK;
  const size_t es = elem_size(d->dtype);
  const size_t nq = BH * d->N * d->dk * es, nv = BH * d->N * d->dv * es;
  const size_t nS = BH * d->dk * d->dv * 4, nz = BH * d->dk * 4;
  if (d->N > 0 && (!q || !k || !v || !out)) return LINATTN_ERR_INVALID;
  if ((S_init == nullptr) != (z_init == nullptr)) return LINATTN_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
      !aligned16(S_final) || !aligned16(z_final) || !aligned16(lambda) || !aligned16(S_init) ||
      !aligned16(z_init))
    return LINATTN_ERR_INVALID;
  if (overlaps(out, nv, q, nq) || overlaps(out, nv, k, nq) || overlaps(out, nv, v, nv) ||
      overlaps(S_final, nS, out, nv) || overlaps(z_final, nz, out, nv) ||
      overlaps(S_final, nS, z_final, nz))
    return LINATTN_ERR_INVALID;
  // the starting state is read while the outputs are written: no overlap
  if (overlaps(S_init, nS, out, nv) || overlaps(S_init, nS, S_final, nS) ||
      overlaps(S_init, nS, z_final, nz) || overlaps(z_init, nz, out, nv) ||
      overlaps(z_init, nz, S_final, nS) || overlaps(z_init, nz, z_final, nz))
    return LINATTN_ERR_INVALID;
  if (d->N == 0) {
    // no token: the final state is the starting state
    if (S_final) {
      const cudaError_t e = S_init ? cudaMemcpyAsync(S_final, S_init, nS, cudaMemcpyDeviceToDevice, s)
                                   : cudaMemsetAsync(S_final, 0, nS, s);
      if (e != cudaSuccess) return LINATTN_ERR_CUDA;
    }
    if (z_final) {
      const cudaError_t e = z_init ? cudaMemcpyAsync(z_final, z_init, nz, cudaMemcpyDeviceToDevice, s)
                                   : cudaMemsetAsync(z_final, 0, nz, s);
      if (e != cudaSuccess) return LINATTN_ERR_CUDA;
    }
    return LINATTN_OK;
  }
  const CausalPath path = causal_path(d);
  if (path == CausalPath::kPairedTc)
    return launch_causal_tc(d, q, k, v, lambda, eps, S_init, z_init, out, S_final, z_final, s);
  // the segment-parallel form when it pays and the workspace holds it
  auto ws_ok = [&](size_t need) -> int {
    if (!aligned16(ws)) return LINATTN_ERR_INVALID;
    if (overlaps(ws, need, q, nq) || overlaps(ws, need, k, nq) || overlaps(ws, need, v, nv) ||
        overlaps(ws, need, out, nv) || overlaps(ws, need, S_final, nS) ||
        overlaps(ws, need, z_final, nz) || overlaps(ws, need, S_init, nS) ||
        overlaps(ws, need, z_init, nz))
      return LINATTN_ERR_INVALID;
    return LINATTN_OK;
  };
  if (path == CausalPath::kSegTc) {
    TcSegments tsg = plan_tc_segments(d);
    const size_t need = tc_segment_bytes(d, tsg);
    if (tsg.G > 1 && ws && ws_bytes >= need) {
      if ((rc = ws_ok(need)) != LINATTN_OK) return rc;
    } else {
      tsg = TcSegments{1, d->N};
    }
    return launch_causal_seg_tc(d, q, k, v, lambda, eps, S_init, z_init, out, S_final, z_final,
                                tsg, static_cast<float *>(tsg.G > 1 ? ws : nullptr), s);
  }
  Segments sg = plan_segments(d);
  const size_t need = segment_bytes(d, sg);
  if (sg.G > 1 && ws && ws_bytes >= need) {
    if ((rc = ws_ok(need)) != LINATTN_OK) return rc;
    sg.ws = static_cast<float *>(ws);
  } else {
    sg = Segments{1, d->N, nullptr};
  }
  if (d->dtype == LINATTN_F32)
    return causal_simt_dispatch<float>(d, q, k, v, lambda, eps, S_init, z_init, out, S_final,
                                       z_final, sg, s);
  return causal_simt_dispatch<bf16>(d, q, k, v, lambda, eps, S_init, z_init, out, S_final,
                                    z_final, sg, s);
}

// Scratch of the no-allocation entry point: a static device array (one per
// device the library is loaded on), its address looked up once per device.
constexpr size_t kScratchBytes = size_t(16) << 20;
__device__ __align__(256) unsigned char g_causal_scratch[kScratchBytes];

// The current context, through the driver entry point (nullptr if unknown).
using CtxGetCurrent = CUresult (*)(CUcontext *);
CUcontext current_context() {
  static CtxGetCurrent fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrent>(p);
  });
  CUcontext c = nullptr;
  if (!fn || fn(&c) != CUDA_SUCCESS) return nullptr;
  return c;
}

// Looked up once per device and context: a context created anew on the
// device (after cudaDeviceReset, say) loads the module again, and the array
// may then sit at another address.
void *scratch_address() {
  static void *addr[64] = {};
  static CUcontext ctx[64] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  const CUcontext cur = current_context();
  if (addr[dev] && cur && ctx[dev] == cur) return addr[dev];
  void *a = nullptr;
  if (cudaGetSymbolAddress(&a, g_causal_scratch) != cudaSuccess) a = nullptr;
  addr[dev] = a;
  ctx[dev] = current_context();   // the lookup makes the device's context current
  return a;
}

}  // namespace
}  // namespace linattn

extern "C" int linattn_fwd_causal(const linattn_dims *d, const void *q, const void *k,
                                  const void *v, const float *lambda, float eps, void *out,
                                  float *S_final, float *z_final, linattn_stream_t stream) {
  return fwd_causal_impl(d, q, k, v, lambda, eps, nullptr, nullptr, out, S_final, z_final,
                         nullptr, 0, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int linattn_fwd_causal_from(const linattn_dims *d, const void *q, const void *k,
                                       const void *v, const float *lambda, float eps,
                                       const float *S_init, const float *z_init, void *out,
                                       float *S_final, float *z_final, linattn_stream_t stream) {
  return fwd_causal_impl(d, q, k, v, lambda, eps, S_init, z_init, out, S_final, z_final,
                         nullptr, 0, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" size_t linattn_fwd_causal_workspace(const linattn_dims *d) {
  if (check_dims(d, true) != LINATTN_OK || d->B == 0 || d->H == 0 || d->N == 0) return 0;
  switch (causal_path(d)) {
    case CausalPath::kSegTc: return tc_segment_bytes(d, plan_tc_segments(d));
    case CausalPath::kPairedTc: return 0;
    case CausalPath::kSimt: break;
  }
  return segment_bytes(d, plan_segments(d));
}

extern "C" int linattn_set_kernel_choice(int op, int kernel, int segments) {
  if (op < LINATTN_OP_CAUSAL || op > LINATTN_OP_BACKWARD) return LINATTN_ERR_INVALID;
  if (kernel < LINATTN_KERNEL_AUTO || kernel > LINATTN_KERNEL_TC_PAIRED) return LINATTN_ERR_INVALID;
  if (kernel == LINATTN_KERNEL_TC_PAIRED && op != LINATTN_OP_CAUSAL) return LINATTN_ERR_INVALID;
  if (segments < 0 || segments > kMaxSegments) return LINATTN_ERR_INVALID;
  g_choice[op].store(kernel, std::memory_order_relaxed);
  if (op == LINATTN_OP_CAUSAL) g_forced_segments.store(segments, std::memory_order_relaxed);
  return LINATTN_OK;
}

extern "C" int linattn_fwd_causal_ws(const linattn_dims *d, const void *q, const void *k,
                                     const void *v, const float *lambda, float eps,
                                     const float *S_init, const float *z_init, void *out,
                                     float *S_final, float *z_final, void *workspace,
                                     size_t workspace_bytes, linattn_stream_t stream) {
  return fwd_causal_impl(d, q, k, v, lambda, eps, S_init, z_init, out, S_final, z_final,
                         workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int linattn_fwd_causal_noalloc(const linattn_dims *d, const void *q, const void *k,
                                          const void *v, const float *lambda, float eps,
                                          void *out, float *S_final, float *z_final,
                                          linattn_stream_t stream) {
  void *ws = scratch_address();
  return fwd_causal_impl(d, q, k, v, lambda, eps, nullptr, nullptr, out, S_final, z_final, ws,
                         ws ? kScratchBytes : 0, reinterpret_cast<cudaStream_t>(stream));
}

namespace linattn {
namespace {

template <int DK, int DVS, typename T>
int launch_state_simt(const linattn_dims *d, const void *k, const void *v, const float *lam,
                      float *S, float *z, cudaStream_t s) {
  const int ctas = d->B * d->H * (d->dv / DVS);
  causal_seg_state_kernel<DK, DVS, T><<<dim3(ctas, 1), 256, 0, s>>>(
      static_cast<const T *>(k), static_cast<const T *>(v), lam, S, z, d->H, d->N, d->dv, d->N,
      1, ident(d));
  return launch_status();
}

template <typename T>
int state_simt_dispatch(const linattn_dims *d, const void *k, const void *v, const float *lam,
                        float *S, float *z, cudaStream_t s) {
  const bool narrow = d->dv == 16;
#define LINATTN_STATE_CASE(DKV)                                                              \
  case DKV:                                                                                 \
    return narrow ? launch_state_simt<DKV, 16, T>(d, k, v, lam, S, z, s)                    \
                  : launch_state_simt<DKV, 32, T>(d, k, v, lam, S, z, s);
  switch (d->dk) {
    LINATTN_STATE_CASE(16)
    LINATTN_STATE_CASE(32)
    LINATTN_STATE_CASE(64)
    LINATTN_STATE_CASE(128)
  }
#undef LINATTN_STATE_CASE
  return LINATTN_ERR_UNSUPPORTED;
}

template <int DKP, int DVP>
int launch_state_tc(const linattn_dims *d, const CUtensorMap &mk, const CUtensorMap &mv,
                    const float *lam, float *S, float *z, cudaStream_t s) {
  auto *sk = stc::causal_seg_state_tc_kernel<DKP, DVP>;
  if (!set_smem(sk, static_cast<int>(stc::sp::kSmemBytes))) return LINATTN_ERR_CUDA;
  sk<<<d->B * d->H, stc::sp::NT, stc::sp::kSmemBytes, s>>>(mk, mv, lam, S, z, d->H, d->N, d->N,
                                                            1, 1, ident(d));
  return launch_status();
}

}  // namespace
}  // namespace linattn

extern "C" int linattn_causal_state(const linattn_dims *d, const void *k, const void *v,
                                    const float *lambda, float *S, float *z,
                                    linattn_stream_t stream) {
  int rc = check_dims(d, true);
  if (rc != LINATTN_OK) return rc;
  const size_t BH = static_cast<size_t>(d->B) * d->H;
  if (BH == 0) return LINATTN_OK;
  const size_t es = elem_size(d->dtype);
  const size_t nk = BH * d->N * d->dk * es, nv = BH * d->N * d->dv * es;
  const size_t nS = BH * d->dk * d->dv * 4, nz = BH * d->dk * 4;
  if (!S || !z || (d->N > 0 && (!k || !v))) return LINATTN_ERR_INVALID;
  if (!aligned16(k) || !aligned16(v) || !aligned16(S) || !aligned16(z) || !aligned16(lambda))
    return LINATTN_ERR_INVALID;
  if (overlaps(S, nS, k, nk) || overlaps(S, nS, v, nv) || overlaps(z, nz, k, nk) ||
      overlaps(z, nz, v, nv) || overlaps(S, nS, z, nz))
    return LINATTN_ERR_INVALID;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (d->N == 0) {
    if (cudaMemsetAsync(S, 0, nS, s) != cudaSuccess || cudaMemsetAsync(z, 0, nz, s) != cudaSuccess)
      return LINATTN_ERR_CUDA;
    return LINATTN_OK;
  }
  if (causal_path(d) != CausalPath::kSimt) {
    const int BHi = d->B * d->H;
    CUtensorMap mk, mv;
    if (!make_map_bf16(&mk, k, d->dk, d->N, BHi) || !make_map_bf16(&mv, v, d->dv, d->N, BHi))
      return LINATTN_ERR_CUDA;
    if (d->dk == 128)
      return d->dv == 128 ? launch_state_tc<2, 2>(d, mk, mv, lambda, S, z, s)
                          : launch_state_tc<2, 1>(d, mk, mv, lambda, S, z, s);
    return d->dv == 128 ? launch_state_tc<1, 2>(d, mk, mv, lambda, S, z, s)
                        : launch_state_tc<1, 1>(d, mk, mv, lambda, S, z, s);
  }
  if (d->dtype == LINATTN_F32) return state_simt_dispatch<float>(d, k, v, lambda, S, z, s);
  return state_simt_dispatch<bf16>(d, k, v, lambda, S, z, s);
}

extern "C" int linattn_combine_states(const linattn_dims *d, int G, const float *lambda,
                                      const float *S_init, const float *z_init, float *dS,
                                      float *dz, linattn_stream_t stream) {
  if (!d || d->B < 0 || d->H < 0 || d->N < 0 || G < 0) return LINATTN_ERR_INVALID;
  if (!supported_dim(d->dk) || !supported_dim(d->dv)) return LINATTN_ERR_UNSUPPORTED;
  if (G > kMaxSegments) return LINATTN_ERR_UNSUPPORTED;
  const size_t BH = static_cast<size_t>(d->B) * d->H;
  if (BH == 0 || G == 0) return LINATTN_OK;
  if (static_cast<long long>(BH) * G * d->dk * d->dv >= (1ll << 31)) return LINATTN_ERR_UNSUPPORTED;
  if ((S_init == nullptr) != (z_init == nullptr) || !dS || !dz) return LINATTN_ERR_INVALID;
  if (!aligned16(dS) || !aligned16(dz) || !aligned16(S_init) || !aligned16(z_init) ||
      !aligned16(lambda))
    return LINATTN_ERR_INVALID;
  const size_t nS = BH * d->dk * d->dv * 4, nz = BH * d->dk * 4;
  if (overlaps(dS, G * nS, dz, G * nz) || overlaps(S_init, nS, dS, G * nS) ||
      overlaps(S_init, nS, dz, G * nz) || overlaps(z_init, nz, dS, G * nS) ||
      overlaps(z_init, nz, dz, G * nz))
    return LINATTN_ERR_INVALID;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int eblocks = (d->dk * d->dv + d->dk + 255) / 256;
  // every segment is N tokens long here: the decay between slots is lambda^N
  causal_seg_combine_kernel<<<dim3(static_cast<unsigned>(BH), eblocks), 256, 0, s>>>(
      lambda, S_init, z_init, dS, dz, d->H, d->dk, d->dv, static_cast<long>(G) * d->N, d->N, G,
      true);
  return launch_status();
}

namespace linattn {
namespace {

int bwd_causal_impl(const linattn_dims *d, const void *q, const void *k, const void *v,
                    const float *lambda, float eps, const void *dy, void *dq, void *dk, void *dv,
                    float *dlambda, void *ws, size_t ws_bytes, bool may_alloc, cudaStream_t s) {
  int rc = check_dims(d, true);
  if (rc != LINATTN_OK) return rc;
  if (bad_eps(eps)) return LINATTN_ERR_INVALID;
  const size_t BH = static_cast<size_t>(d->B) * d->H;
  const size_t es = elem_size(d->dtype);
  const size_t nq = BH * d->N * d->dk * es, nv = BH * d->N * d->dv * es;
  const size_t nl = static_cast<size_t>(d->H) * 4;
  if (BH > 0 && d->N > 0 && (!q || !k || !v || !dy || !dq || !dk || !dv))
    return LINATTN_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dy) || !aligned16(dq) ||
      !aligned16(dk) || !aligned16(dv) || !aligned16(lambda) || !aligned16(dlambda) ||
      !aligned16(ws))
    return LINATTN_ERR_INVALID;
  // every output (and the workspace) overlaps no input and no other output
  const void *in[5] = {q, k, v, dy, lambda};
  const size_t nin[5] = {nq, nq, nv, nv, nl};
  const void *outp[5] = {dq, dk, dv, dlambda, ws};
  const size_t nout[5] = {nq, nq, nv, nl, ws ? ws_bytes : 0};
  for (int o = 0; o < 5; ++o) {
    for (int i = 0; i < 5; ++i)
      if (overlaps(outp[o], nout[o], in[i], nin[i])) return LINATTN_ERR_INVALID;
    for (int o2 = o + 1; o2 < 5; ++o2)
      if (overlaps(outp[o], nout[o], outp[o2], nout[o2])) return LINATTN_ERR_INVALID;
  }
  if (dlambda && cudaMemsetAsync(dlambda, 0, nl, s) != cudaSuccess) return LINATTN_ERR_CUDA;
  if (BH == 0 || d->N == 0) return LINATTN_OK;
  if (use_tc_bwd(d))
    return launch_bwd_tc(d, q, k, v, lambda, eps, dy, dq, dk, dv, dlambda, ws, ws_bytes,
                         may_alloc, s);
  if (d->dtype == LINATTN_F32)
    return causal_bwd_dispatch<float>(d, q, k, v, lambda, eps, dy, dq, dk, dv, dlambda, s);
  return causal_bwd_dispatch<bf16>(d, q, k, v, lambda, eps, dy, dq, dk, dv, dlambda, s);
}

}  // namespace
}  // namespace linattn

extern "C" int linattn_bwd_causal(const linattn_dims *d, const void *q, const void *k,
                                  const void *v, const float *lambda, float eps, const void *dy,
                                  void *dq, void *dk, void *dv, float *dlambda,
                                  linattn_stream_t stream) {
  return bwd_causal_impl(d, q, k, v, lambda, eps, dy, dq, dk, dv, dlambda, nullptr, 0, true,
                         reinterpret_cast<cudaStream_t>(stream));
}

extern "C" size_t linattn_bwd_causal_workspace(const linattn_dims *d) {
  if (!d || check_dims(d, true) != LINATTN_OK || !use_tc_bwd(d)) return 0;
  if (static_cast<size_t>(d->B) * d->H == 0 || d->N == 0) return 0;
  return bwd_tc_bytes(d, bwd_split(d));
}

extern "C" int linattn_bwd_causal_ws(const linattn_dims *d, const void *q, const void *k,
                                     const void *v, const float *lambda, float eps,
                                     const void *dy, void *dq, void *dk, void *dv,
                                     float *dlambda, void *workspace, size_t workspace_bytes,
                                     linattn_stream_t stream) {
  if (!workspace && workspace_bytes) return LINATTN_ERR_INVALID;
  return bwd_causal_impl(d, q, k, v, lambda, eps, dy, dq, dk, dv, dlambda, workspace,
                         workspace ? workspace_bytes : 0, false,
                         reinterpret_cast<cudaStream_t>(stream));
}

namespace linattn {
namespace {

// Both global entry points: d->N queries against Nk keys/values.
int fwd_global_impl(const linattn_dims *d, int Nk, const void *q, const void *k, const void *v,
                    const uint8_t *kpm, float eps, void *out, float *KV, float *ksum,
                    cudaStream_t s) {
  int rc = check_dims(d, true);
  if (rc != LINATTN_OK) return rc;
  if (Nk < 0) return LINATTN_ERR_INVALID;
  if (Nk > 0) {
    linattn_dims dk_ = *d;
    dk_.N = Nk;
    if ((rc = check_dims(&dk_, true)) != LINATTN_OK) return rc;
  }
  if (bad_eps(eps)) return LINATTN_ERR_INVALID;
  const size_t BH = static_cast<size_t>(d->B) * d->H;
  if (BH == 0) return LINATTN_OK;
  if (!KV || !ksum) return LINATTN_ERR_INVALID;
  const size_t es = elem_size(d->dtype);
  const size_t nq = BH * d->N * d->dk * es, ny = BH * d->N * d->dv * es;
  const size_t nk = BH * Nk * d->dk * es, nv = BH * Nk * d->dv * es;
  const size_t nS = BH * d->dk * d->dv * 4, nz = BH * d->dk * 4;
  if ((d->N > 0 && (!q || !out)) || (Nk > 0 && (!k || !v))) return LINATTN_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(KV) ||
      !aligned16(ksum))
    return LINATTN_ERR_INVALID;
  if (overlaps(out, ny, q, nq) || overlaps(out, ny, k, nk) || overlaps(out, ny, v, nv) ||
      overlaps(KV, nS, out, ny) || overlaps(ksum, nz, out, ny) || overlaps(KV, nS, ksum, nz) ||
      overlaps(KV, nS, k, nk) || overlaps(KV, nS, v, nv) || overlaps(KV, nS, q, nq) ||
      overlaps(ksum, nz, q, nq) || overlaps(ksum, nz, k, nk) || overlaps(ksum, nz, v, nv))
    return LINATTN_ERR_INVALID;
  // the padding mask is read while the outputs are written: no overlap
  const size_t nm = kpm ? static_cast<size_t>(d->B) * Nk : 0;
  if (overlaps(kpm, nm, out, ny) || overlaps(kpm, nm, KV, nS) || overlaps(kpm, nm, ksum, nz))
    return LINATTN_ERR_INVALID;
  if ((rc = zero_kv(KV, nS, ksum, nz, s)) != LINATTN_OK) return rc;
  if (d->N == 0 && Nk == 0) return LINATTN_OK;
  if (use_tc_global(d)) return launch_global_tc(d, Nk, q, k, v, kpm, eps, out, KV, ksum, s);
  if (d->dtype == LINATTN_F32)
    return global_dispatch<float>(d, Nk, q, k, v, kpm, eps, out, KV, ksum, s);
  return global_dispatch<bf16>(d, Nk, q, k, v, kpm, eps, out, KV, ksum, s);
}

}  // namespace
}  // namespace linattn

extern "C" int linattn_fwd_global(const linattn_dims *d, const void *q, const void *k,
                                  const void *v, float eps, void *out, float *KV, float *ksum,
                                  linattn_stream_t stream) {
  return fwd_global_impl(d, d ? d->N : 0, q, k, v, nullptr, eps, out, KV, ksum,
                         reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int linattn_fwd_global_cross(const linattn_dims *d, int Nk, const void *q,
                                        const void *k, const void *v, float eps, void *out,
                                        float *KV, float *ksum, linattn_stream_t stream) {
  return fwd_global_impl(d, Nk, q, k, v, nullptr, eps, out, KV, ksum,
                         reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int linattn_fwd_global_masked(const linattn_dims *d, int Nk, const void *q,
                                         const void *k, const void *v,
                                         const unsigned char *key_padding_mask, float eps,
                                         void *out, float *KV, float *ksum,
                                         linattn_stream_t stream) {
  return fwd_global_impl(d, Nk, q, k, v, key_padding_mask, eps, out, KV, ksum,
                         reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int linattn_decode_step(const linattn_dims *d, const void *q, const void *k,
                                   const void *v, const float *lambda, float eps, float *S,
                                   float *z, void *out, linattn_stream_t stream) {
  int rc = check_dims(d, false);
  if (rc != LINATTN_OK) return rc;
  if (bad_eps(eps)) return LINATTN_ERR_INVALID;
  const size_t BH = static_cast<size_t>(d->B) * d->H;
  if (BH == 0) return LINATTN_OK;
  if (!q || !k || !v || !S || !z || !out) return LINATTN_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(S) || !aligned16(z) ||
      !aligned16(out) || !aligned16(lambda))
    return LINATTN_ERR_INVALID;
  const size_t es = elem_size(d->dtype);
  const size_t nq = BH * d->dk * es, nv = BH * d->dv * es;
  const size_t nS = BH * d->dk * d->dv * 4, nz = BH * d->dk * 4;
  if (overlaps(out, nv, q, nq) || overlaps(out, nv, k, nq) || overlaps(out, nv, v, nv) ||
      overlaps(S, nS, out, nv) || overlaps(z, nz, out, nv) || overlaps(S, nS, z, nz) ||
      overlaps(S, nS, q, nq) || overlaps(S, nS, k, nq) || overlaps(S, nS, v, nv))
    return LINATTN_ERR_INVALID;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (d->dtype == LINATTN_F32)
    return decode_dispatch<float>(d, q, k, v, lambda, eps, S, z, out, s);
  return decode_dispatch<bf16>(d, q, k, v, lambda, eps, S, z, out, s);
}

// ------------------------------------------------------------ Performer features
namespace {

bool supported_features(int m) { return m == 8 || m == 16 || m == 32 || m == 64; }

// bf16 with d in {64, 128} and m in {32, 64} takes the tensor-core kernel;
// LINATTN_KERNEL_CUDA_CORES chosen for the feature map forces the CUDA-core
// kernel.
bool use_tc_features(int d, int m, int dtype) {
  if (choice(LINATTN_OP_PERFORMER) == LINATTN_KERNEL_CUDA_CORES) return false;
  return dtype == LINATTN_BF16 && (d == 64 || d == 128) && (m == 32 || m == 64);
}

template <int D, int M>
int launch_features_tc(long long rows, int kernel, const void *x, const void *omega, void *out,
                       cudaStream_t s) {
  using L = perf::Layout<D, M>;
  auto *kern = performer_tc_kernel<D, M>;
  if (!set_smem(kern, static_cast<int>(L::kSmem))) return LINATTN_ERR_CUDA;
  const int sms = num_sms();
  if (sms <= 0) return LINATTN_ERR_CUDA;
  CUtensorMap mx, mw, my;
  const int r = static_cast<int>(rows);
  if (!make_map_bf16(&mx, x, D, r, 1) || !make_map_bf16(&mw, omega, D, M, 1, M) ||
      !make_map_bf16(&my, out, 2 * M, r, 1, 32))   // 32-row slabs, one per quadrant team
    return LINATTN_ERR_CUDA;
  const long long tiles = (rows + perf::R - 1) / perf::R;
  const int grid = static_cast<int>(tiles < sms ? tiles : sms);
  kern<<<grid, perf::NT, L::kSmem, s>>>(mx, mw, my, static_cast<long>(rows), kernel);
  return launch_status();
}

template <typename T>
int launch_features_simt(long long rows, int d, int m, int kernel, const void *x,
                         const void *omega, void *out, cudaStream_t s) {
  const int sms = num_sms();
  if (sms <= 0) return LINATTN_ERR_CUDA;
  const int bytes = (m * (d + 1) + (kPerfSimtThreads / 32) * d) * 4;
  const long long want = (rows + kPerfSimtThreads / 32 - 1) / (kPerfSimtThreads / 32);
  const int grid = static_cast<int>(want < 8LL * sms ? want : 8LL * sms);
  performer_simt_kernel<T><<<grid, kPerfSimtThreads, bytes, s>>>(
      static_cast<const T *>(x), static_cast<const T *>(omega), static_cast<T *>(out),
      static_cast<long>(rows), d, m, kernel);
  return launch_status();
}

}  // namespace

extern "C" int linattn_performer_features(long long rows, int d, int m, int kernel, int dtype,
                                          const void *x, const void *omega, void *out,
                                          linattn_stream_t stream) {
  if (rows < 0) return LINATTN_ERR_INVALID;
  if (dtype != LINATTN_BF16 && dtype != LINATTN_F32) return LINATTN_ERR_UNSUPPORTED;
  if (kernel != LINATTN_PERFORMER_SOFTMAX && kernel != LINATTN_PERFORMER_GAUSSIAN)
    return LINATTN_ERR_UNSUPPORTED;
  if (!supported_dim(d) || !supported_features(m)) return LINATTN_ERR_UNSUPPORTED;
  if (rows * (d > 2 * m ? d : 2 * m) >= (1LL << 31)) return LINATTN_ERR_UNSUPPORTED;
  if (rows == 0) return LINATTN_OK;   // nothing to read or write: NULL buffers allowed
  if (!x || !omega || !out) return LINATTN_ERR_INVALID;
  if (!aligned16(x) || !aligned16(omega) || !aligned16(out)) return LINATTN_ERR_INVALID;
  const size_t es = elem_size(dtype);
  const size_t nx = static_cast<size_t>(rows) * d * es, nw = static_cast<size_t>(m) * d * es;
  const size_t ny = static_cast<size_t>(rows) * 2 * m * es;
  if (overlaps(out, ny, x, nx) || overlaps(out, ny, omega, nw)) return LINATTN_ERR_INVALID;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (use_tc_features(d, m, dtype)) {
    if (d == 64) return m == 32 ? launch_features_tc<64, 32>(rows, kernel, x, omega, out, s)
                                : launch_features_tc<64, 64>(rows, kernel, x, omega, out, s);
    return m == 32 ? launch_features_tc<128, 32>(rows, kernel, x, omega, out, s)
                   : launch_features_tc<128, 64>(rows, kernel, x, omega, out, s);
  }
  if (dtype == LINATTN_F32)
    return launch_features_simt<float>(rows, d, m, kernel, x, omega, out, s);
  return launch_features_simt<bf16>(rows, d, m, kernel, x, omega, out, s);
}

extern "C" const char *linattn_status_string(int status) {
  switch (status) {
    case LINATTN_OK: return "ok";
    case LINATTN_ERR_INVALID: return "invalid argument (NULL, negative, misaligned or aliased)";
    case LINATTN_ERR_UNSUPPORTED: return "unsupported size or dtype";
    case LINATTN_ERR_CUDA: return "CUDA runtime error at launch";
    case LINATTN_ERR_DEVICE: return "a kernel recorded a device-side error";
  }
  return "unknown status";
}

extern "C" int linattn_device_status(int clear, linattn_stream_t stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return -1;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(v)) != cudaSuccess) return -1;
  if (clear) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(g_status, &zero, sizeof(zero)) != cudaSuccess) return -1;
  }
  return static_cast<int>(v);
}

extern "C" int linattn_version(void) { return kVersion; }
