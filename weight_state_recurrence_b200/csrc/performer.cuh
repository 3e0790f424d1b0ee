// Performer random features (linear-attention note §4.2): for a projection
// Omega [m, d] with rows omega_l,
//   phi(x) = g(x)/sqrt(m) [cos(omega_1.x) .. cos(omega_m.x), sin(omega_1.x) .. sin(omega_m.x)]
// with g(x) = exp(|x|^2/2) (h = 1: phi(x).phi(y) estimates exp(x.y)) or
// g(x) = 1 (h(x) = exp(-|x|^2/2): it estimates exp(-|x-y|^2/2)).  The rows of
// the output are the feature vectors the attention kernels take in identity
// mode (d_k = 2m).
//
//   performer_tc_kernel    bf16, d in {64, 128}, m in {32, 64}.  U = X Omega^T
//                          is a dense contraction, so it runs on the tensor
//                          cores: 128-row tiles of X arrive by TMA, one
//                          M = 128, N = m, K = d chain per tile accumulates
//                          in TMEM (two buffers), and sixteen epilogue warps
//                          turn U into cos/sin, scale by g/sqrt(m) and send
//                          the bf16 tile out by TMA.  The four warps of a TMEM
//                          lane quadrant own its 32 rows (a quarter of the
//                          columns each) and work as an independent team:
//                          they meet only at their own named barrier and store
//                          their own 32-row slab.  Persistent CTAs.
//   performer_simt_kernel  every other case, fp32 arithmetic with the
//                          accurate sincosf/expf: one warp per row.
#pragma once
#include "common.cuh"
#include "sm100.cuh"

namespace linattn {

enum : int { kPerfSoftmax = 0, kPerfGaussian = 1 };

// sin and cos of u for the bf16 path, on the FMA pipe (the special-function
// pipe, shared by the sin/cos approximations, float rounding and conversions,
// is otherwise the bottleneck of the epilogue), scaled by sc:
//   u = j pi + r:  j = u / pi rounded to nearest by adding 1.5 * 2^23 (the
//     sum's lowest mantissa bit is then j's parity), r by Cody and Waite's
//     two-constant reduction with pi = P1 + P2, P1 = 3.140625 (8 significant
//     bits: j P1 is exact for |j| < 2^16, so |u| up to about 2e5 reduces
//     accurately);
//   sin r, cos r by their Taylor series through r^9 and r^8 on |r| <= pi/2
//     (truncation errors below 4e-6 and 2.5e-5, against the 2^-9 relative
//     rounding of the bf16 result);
//   sin u = (-1)^j sin r, cos u = (-1)^j cos r: the sign goes into sc.
__device__ __forceinline__ void sincos_poly(float u, float sc, float *sn, float *cs) {
  const float kRound = 12582912.f;                            // 1.5 * 2^23
  const float t = fmaf(u, 0.318309886183790672f, kRound);    // u / pi + 1.5 * 2^23
  const float jf = t - kRound;
  float r = fmaf(-jf, 3.140625f, u);
  r = fmaf(-jf, 9.67653589793116e-4f, r);                    // pi - 3.140625
  const float sg = __int_as_float(__float_as_int(sc) ^ (__float_as_int(t) << 31));
  const float r2 = r * r;
  float ps = fmaf(r2, 2.75573192239858907e-6f, -1.98412698412698413e-4f);   // 1/9!, -1/7!
  ps = fmaf(r2, ps, 8.33333333333333333e-3f);                               // 1/5!
  ps = fmaf(r2, ps, -0.166666666666666667f);                                // -1/3!
  ps = fmaf(r2, ps, 1.0f);
  float pc = fmaf(r2, 2.48015873015873016e-5f, -1.38888888888888889e-3f);   // 1/8!, -1/6!
  pc = fmaf(r2, pc, 4.16666666666666667e-2f);                               // 1/4!
  pc = fmaf(r2, pc, -0.5f);
  pc = fmaf(r2, pc, 1.0f);
  *sn = (r * sg) * ps;
  *cs = sg * pc;
}

// ----------------------------------------------------------- CUDA cores
constexpr int kPerfSimtThreads = 256;

template <typename T>
__global__ void __launch_bounds__(kPerfSimtThreads) performer_simt_kernel(
    const T *__restrict__ x, const T *__restrict__ omega, T *__restrict__ out, long rows, int d,
    int m, int kernel) {
  extern __shared__ float psm[];
  const int WS = d + 1;                       // padded omega rows: lanes walk rows
  float *sW = psm;                            // [m][d+1]
  float *sX = sW + m * WS;                    // [8 warps][d]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int i = tid; i < m * d; i += kPerfSimtThreads) sW[(i / d) * WS + i % d] = to_f32(omega[i]);
  __syncthreads();
  float *xr = sX + warp * d;
  const float inv_sqrt_m = rsqrtf(static_cast<float>(m));
  const long nwarps = static_cast<long>(gridDim.x) * (kPerfSimtThreads / 32);
  for (long r = static_cast<long>(blockIdx.x) * (kPerfSimtThreads / 32) + warp; r < rows;
       r += nwarps) {
    float n2 = 0.f;
    for (int c = lane; c < d; c += 32) {
      const float a = to_f32(x[r * d + c]);
      xr[c] = a;
      n2 = fmaf(a, a, n2);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) n2 += __shfl_xor_sync(0xffffffffu, n2, o);
    __syncwarp();
    const float sc = (kernel == kPerfSoftmax ? expf(0.5f * n2) : 1.f) * inv_sqrt_m;
    T *orow = out + r * 2 * m;
    for (int l = lane; l < m; l += 32) {
      float u = 0.f;
      for (int c = 0; c < d; ++c) u = fmaf(sW[l * WS + c], xr[c], u);
      float s, co;
      sincosf(u, &s, &co);
      orow[l] = from_f32<T>(co * sc);
      orow[m + l] = from_f32<T>(s * sc);
    }
    __syncwarp();
  }
}

// --------------------------------------------------------- tensor cores
namespace perf {
constexpr int R = 128;                   // rows per tile (the MMA's M)
constexpr int kStages = 4;               // X tile ring
constexpr uint32_t kPanel = R * 128;     // 128 rows x 64 bf16, 128B-swizzled
constexpr int kGroups = 4;               // epilogue threads per row (warps per quadrant)
constexpr int kEpi = kGroups * R;        // epilogue threads (warps 4 .. 4 + kEpi/32 - 1)
constexpr int NT = 128 + kEpi;           // warp 0 TMA, warp 1 MMA, warps 2-3 idle
enum { kXFull = 0, kXEmpty = kStages, kAccFull = 2 * kStages, kAccEmpty = kAccFull + 2,
       kWFull = kAccEmpty + 2, kFinal, kNumBars };

template <int D, int M>
struct Layout {
  static_assert((D == 64 || D == 128) && (M == 32 || M == 64), "tensor-core feature shapes");
  static constexpr uint32_t kXStage = (D / 64) * kPanel;
  static constexpr uint32_t kOffX = 0;
  static constexpr uint32_t kOffW = kOffX + kStages * kXStage;     // D/64 panels of M rows
  static constexpr uint32_t kWPanel = M * 128;
  static constexpr uint32_t kOffY = kOffW + (D / 64) * kWPanel;    // 2 staging tiles
  static constexpr uint32_t kYStage = (2 * M / 64) * kPanel;
  static constexpr uint32_t kOffMisc = kOffY + 2 * kYStage;
  static constexpr uint32_t kMiscTmem = 8 * kNumBars, kMiscFail = kMiscTmem + 4,
                            kMiscEFail = kMiscTmem + 8;   // 4 ints: one per row quadrant
  static constexpr uint32_t kOffPart = kOffMisc + 256;              // [kGroups][R] |x|^2 parts
  static constexpr uint32_t kSmem = kOffPart + kGroups * R * 4;
  static constexpr uint32_t kTmCols = 2 * M;                        // two accumulators
  static_assert(kOffW % 1024 == 0 && kOffY % 1024 == 0, "swizzled tiles need 1 KB alignment");
  static_assert(kSmem <= 227 * 1024, "shared memory");
};
}  // namespace perf

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&p);
}

template <int D, int M>
__global__ void __launch_bounds__(perf::NT, 1)
    performer_tc_kernel(const __grid_constant__ CUtensorMap tm_x,
                        const __grid_constant__ CUtensorMap tm_w,
                        const __grid_constant__ CUtensorMap tm_y, long rows, int kernel) {
  using namespace perf;
  using L = Layout<D, M>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *sm = smem_raw;
  const uint32_t sb = smem_u32(sm);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (sb & 1023u) {   // the swizzled tiles need a 1 KB aligned base
    if (tid == 0) atomicOr(&g_status, kStatusWaitTimeout);
    return;
  }
  auto bar = [&](int i) { return sb + L::kOffMisc + 8u * static_cast<uint32_t>(i); };
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + L::kOffMisc + L::kMiscTmem);
  volatile int *fail = reinterpret_cast<volatile int *>(sm + L::kOffMisc + L::kMiscFail);
  volatile int *efail = reinterpret_cast<volatile int *>(sm + L::kOffMisc + L::kMiscEFail);

  const long ntiles = (rows + R - 1) / R;
  const long t0 = ntiles * blockIdx.x / gridDim.x, t1 = ntiles * (blockIdx.x + 1) / gridDim.x;
  const int nmine = static_cast<int>(t1 - t0);

  if (tid == 0) {
    // the four quadrant teams each release an X stage and an accumulator
    for (int i = 0; i < kNumBars; ++i)
      mbar_init(bar(i), (i >= kXEmpty && i < kXEmpty + kStages) ||
                                (i >= kAccEmpty && i < kAccEmpty + 2) ? 4 : 1);
    *fail = 0;
    for (int q = 0; q < 4; ++q) efail[q] = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_w);
    tma_prefetch_desc(&tm_y);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), L::kTmCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      mbar_arrive_expect_tx(bar(kWFull), (D / 64) * L::kWPanel);
      for (int p = 0; p < D / 64; ++p)
        tma_load_3d(sb + L::kOffW + p * L::kWPanel, &tm_w, bar(kWFull), 64 * p, 0, 0);
      int issued = 0;
      for (int i = 0; i < nmine && !*fail; ++i) {
        const int s = i % kStages;
        if (i >= kStages && !mbar_wait(bar(kXEmpty + s), ((i / kStages) - 1) & 1)) {
          *fail = 1;
          break;
        }
        const uint32_t b = bar(kXFull + s);
        mbar_arrive_expect_tx(b, L::kXStage);
        const int row0 = static_cast<int>((t0 + i) * R);
        for (int p = 0; p < D / 64; ++p)
          tma_load_3d(sb + L::kOffX + s * L::kXStage + p * kPanel, &tm_x, b, 64 * p, row0, 0);
        issued = i + 1;
      }
      // let the copies still in flight land before the CTA exits
      mbar_wait(bar(kWFull), 0);
      if (*fail)
        for (int i = issued - kStages < 0 ? 0 : issued - kStages; i < issued; ++i)
          mbar_wait(bar(kXFull + i % kStages), (i / kStages) & 1);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issue
    if (lane == 0) {
      const uint32_t id = idesc_bf16(R, M, 0, 0);   // both operands K-major
      bool ok = mbar_wait(bar(kWFull), 0);
      for (int i = 0; i < nmine && ok; ++i) {
        const int s = i % kStages, a = i & 1;
        ok = !*fail && mbar_wait(bar(kXFull + s), (i / kStages) & 1);
        if (ok && i >= 2) ok = mbar_wait(bar(kAccEmpty + a), ((i >> 1) - 1) & 1);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t xa = sb + L::kOffX + s * L::kXStage + (ks >> 2) * kPanel + (ks & 3) * 32;
          const uint32_t wa = sb + L::kOffW + (ks >> 2) * L::kWPanel + (ks & 3) * 32;
          umma_bf16(tmem + a * M, sdesc_sw128(xa, 16, 1024), sdesc_sw128(wa, 16, 1024), id,
                    ks > 0);
        }
        umma_commit(bar(kAccFull + a));
      }
      if (!ok) *fail = 1;
      umma_commit(bar(kFinal));
      mbar_wait(bar(kFinal), 0);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------ epilogue
    // quadrant team q = warp % 4 owns tile rows [32 q, 32 q + 32) (its TMEM
    // lanes); thread (row r, group g) takes columns [g QM, (g+1) QM) of U ->
    // cos at those columns, sin at M + those columns, and a quarter of |x_r|^2
    const int q = warp & 3;
    const int g = (warp - 4) >> 2;
    const int r = q * 32 + lane;
    const bool lead = g == 0 && lane == 0;     // the team's TMA-store / barrier thread
    const uint32_t lf = static_cast<uint32_t>(q * 32) << 16;
    constexpr int QM = M / kGroups;           // 16 or 8 columns of U per thread
    constexpr int QC = D / kGroups / 8;       // 16-byte chunks of x per thread (4 or 2)
    float *part = reinterpret_cast<float *>(sm + L::kOffPart);
    const float inv_sqrt_m = rsqrtf(static_cast<float>(M));
    for (int i = 0; i < nmine; ++i) {
      const int s = i % kStages, a = i & 1;
      const bool ok = !*fail && mbar_wait(bar(kAccFull + a), (i >> 1) & 1);
      if (!ok) efail[q] = 1;
      tc_fence_after();
      if (ok && kernel == kPerfSoftmax) {
        // this thread's part of |x_r|^2 from the staged tile (the MMA has
        // finished reading it)
        const uint8_t *xs = sm + L::kOffX + s * L::kXStage;
        float n2 = 0.f;
#pragma unroll
        for (int j = 0; j < QC; ++j) {
          const int ch = g * QC + j;            // 16-byte chunk of the row
          const uint4 w =
              *reinterpret_cast<const uint4 *>(xs + (ch >> 3) * kPanel + sw128_offset(r, 16 * (ch & 7)));
          const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float lo = __uint_as_float(ww[e] << 16), hi = __uint_as_float(ww[e] & 0xffff0000u);
            n2 = fmaf(lo, lo, n2);
            n2 = fmaf(hi, hi, n2);
          }
        }
        part[g * R + r] = n2;
      }
      // the team's rows of staging tile a must be free: its store of tile i-2
      // has read them
      if (i >= 2 && lead) tma_store_wait_read_1();
      named_bar_sync(1 + q, 32 * kGroups);
      if (efail[q]) break;
      if (lead) mbar_arrive(bar(kXEmpty + s));
      float sc = inv_sqrt_m;
      if (kernel == kPerfSoftmax) {
        float n2 = 0.f;
#pragma unroll
        for (int p = 0; p < kGroups; ++p) n2 += part[p * R + r];
        sc *= expf(0.5f * n2);
      }
      uint32_t u[QM];
      if constexpr (QM == 16) {
        tmem_ld_32x32b_x16(tmem + lf + a * M + g * QM, u);
      } else {
        tmem_ld_32x32b_x8(tmem + lf + a * M + g * QM, u);
      }
      tmem_wait_ld();
      tc_fence_before();
      uint8_t *stg = sm + L::kOffY + a * L::kYStage;
#pragma unroll
      for (int j = 0; j < QM / 8; ++j) {
        uint32_t cw[4], sw[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float s0, c0, s1, c1;
          sincos_poly(__uint_as_float(u[8 * j + 2 * e]), sc, &s0, &c0);
          sincos_poly(__uint_as_float(u[8 * j + 2 * e + 1]), sc, &s1, &c1);
          cw[e] = pack_bf16x2(c0, c1);
          sw[e] = pack_bf16x2(s0, s1);
        }
        const int cc = g * QM + 8 * j;    // cosine column; the sine is at M + cc
        const int sc_col = M + cc;
        *reinterpret_cast<uint4 *>(stg + (cc >> 6) * kPanel + sw128_offset(r, (cc & 63) * 2)) =
            make_uint4(cw[0], cw[1], cw[2], cw[3]);
        *reinterpret_cast<uint4 *>(stg + (sc_col >> 6) * kPanel +
                                   sw128_offset(r, (sc_col & 63) * 2)) =
            make_uint4(sw[0], sw[1], sw[2], sw[3]);
      }
      fence_proxy_async_smem();
      named_bar_sync(1 + q, 32 * kGroups);
      if (lead) {
        mbar_arrive(bar(kAccEmpty + a));
        // the team's 32-row slab of every 64-column panel (4 KB, 1 KB aligned)
        // a slab wholly past the last row is not stored; its (empty) group is
        // still committed so the group count per tile stays one
        const long row0 = (t0 + i) * R + 32 * q;
        if (row0 < rows)
          for (int p = 0; p < 2 * M / 64; ++p)
            tma_store_3d(&tm_y, sb + L::kOffY + a * L::kYStage + p * kPanel + 32 * q * 128,
                         64 * p, static_cast<int>(row0), 0);
        tma_store_commit();
      }
    }
    if (lead) tma_store_wait_all();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmCols);
  }
}

}  // namespace linattn
