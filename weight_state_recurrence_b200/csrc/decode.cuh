// Single-token decode step: one pass over each head's fp32 state.
//
//   S <- lambda S + phi(k) v^T,  z <- lambda z + phi(k),
//   y  = phi(q)^T S / (phi(q)^T z + eps)
// (fast-weight article §4.1 forward_step and §3.1 constant d x d cache;
//  linear-attention note §5 and §6 forward_autoregressive).
//
// The step is bound by HBM traffic on the state: every head reads and writes
// dk*dv*4 bytes of S.  The kernel is persistent (one CTA per SM) and streams
// heads through a ring of shared-memory stages filled by 1-D TMA bulk copies
// (S, z, q, k, v of one head per stage), so two heads are in flight while a
// third is updated.  Each thread owns a float4 column group of dv and a
// strided set of rows; it reads S from shared memory, does the rank-1 update
// and the query read in registers, and writes S back to HBM with streaming
// 128-bit stores.  Column sums of phi(q)^T S are combined across rows through
// shared memory; phi(q)^T z is a warp-shuffle reduction.
#pragma once
#include "common.cuh"
#include "sm100.cuh"

namespace linattn {

constexpr int kDecodeStages = 3;
constexpr int kDecodeThreads = 256;

template <int DK, int DV, typename T>
struct DecodeLayout {
  static constexpr uint32_t kS = DK * DV * 4;
  static constexpr uint32_t kZ = DK * 4;
  static constexpr uint32_t kQ = DK * sizeof(T);
  static constexpr uint32_t kV = DV * sizeof(T);
  static constexpr uint32_t kBytes = kS + kZ + 2 * kQ + kV;          // bulk bytes per head
  static constexpr uint32_t kStage = (kBytes + 127) / 128 * 128;
  static constexpr int TPR = DV / 4;                                  // threads per S row
  static constexpr int RPP = kDecodeThreads / TPR;                    // rows per pass
  static constexpr uint32_t kRed = RPP * DV * 4;                      // partial column sums
  static constexpr uint32_t kSmem = kDecodeStages * kStage + kRed + 2 * DK * 4 + 64 + 128;
};

template <int DK, int DV, typename T>
__global__ void __launch_bounds__(kDecodeThreads, 1) decode_step_kernel(
    const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
    const float *__restrict__ lam, float eps, float *__restrict__ S, float *__restrict__ z,
    T *__restrict__ out, int H, int BH, bool ident) {
  using Lay = DecodeLayout<DK, DV, T>;
  constexpr int NT = kDecodeThreads, TPR = Lay::TPR, RPP = Lay::RPP;
  constexpr int PASSES = (DK + RPP - 1) / RPP;
  static_assert(DV % 4 == 0 && TPR <= NT, "dv must be a multiple of 4");
  static_assert(Lay::kS % 16 == 0 && Lay::kZ % 16 == 0 && Lay::kQ % 16 == 0 && Lay::kV % 16 == 0,
                "bulk copies move multiples of 16 bytes");

  extern __shared__ uint8_t dsm_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dsm_raw) + 127) &
                                            ~static_cast<uintptr_t>(127));
  float *s_red = reinterpret_cast<float *>(sm + kDecodeStages * Lay::kStage);
  float *s_fk = s_red + RPP * DV;
  float *s_fq = s_fk + DK;
  float *s_den = s_fq + DK;                       // NT/32 partials
  uint8_t *bars = reinterpret_cast<uint8_t *>(s_den + 16);
  const uint32_t bar0 = smem_u32(bars);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(bars + 32);

  const int tid = threadIdx.x;
  const int nmine = (BH - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) /
                    static_cast<int>(gridDim.x);

  auto issue = [&](int i) {
    const long p = blockIdx.x + static_cast<long>(i) * gridDim.x;
    const int st = i % kDecodeStages;
    const uint32_t base = smem_u32(sm + st * Lay::kStage);
    const uint32_t bar = bar0 + 8 * st;
    mbar_arrive_expect_tx(bar, Lay::kBytes);
    bulk_load(base, S + p * DK * DV, Lay::kS, bar);
    bulk_load(base + Lay::kS, z + p * DK, Lay::kZ, bar);
    bulk_load(base + Lay::kS + Lay::kZ, q + p * DK, Lay::kQ, bar);
    bulk_load(base + Lay::kS + Lay::kZ + Lay::kQ, k + p * DK, Lay::kQ, bar);
    bulk_load(base + Lay::kS + Lay::kZ + 2 * Lay::kQ, v + p * DV, Lay::kV, bar);
  };

  if (tid == 0) {
    for (int st = 0; st < kDecodeStages; ++st) mbar_init(bar0 + 8 * st, 1);
    *abort_flag = 0;
    fence_mbar_init();
    for (int i = 0; i < nmine && i < kDecodeStages; ++i) issue(i);
  }
  __syncthreads();

  const int c4 = tid % TPR;
  const int r0 = tid / TPR;
  int i = 0;
  for (; i < nmine; ++i) {
    const long p = blockIdx.x + static_cast<long>(i) * gridDim.x;
    const int st = i % kDecodeStages;
    const uint8_t *stage = sm + st * Lay::kStage;
    const float *sS = reinterpret_cast<const float *>(stage);
    const float *sz = reinterpret_cast<const float *>(stage + Lay::kS);
    const T *sq = reinterpret_cast<const T *>(stage + Lay::kS + Lay::kZ);
    const T *sk = reinterpret_cast<const T *>(stage + Lay::kS + Lay::kZ + Lay::kQ);
    const T *sv = reinterpret_cast<const T *>(stage + Lay::kS + Lay::kZ + 2 * Lay::kQ);
    const int h = static_cast<int>(p % H);
    const float L = lam ? lam[h] : 1.f;

    if (!mbar_wait(bar0 + 8 * st, (i / kDecodeStages) & 1)) *abort_flag = 1;
    __syncthreads();
    if (*abort_flag) break;

    float part = 0.f;
    if (tid < DK) {
      const float fk = feat_f32(to_f32(sk[tid]), ident);
      const float fq = feat_f32(to_f32(sq[tid]), ident);
      s_fk[tid] = fk;
      s_fq[tid] = fq;
      const float zn = fmaf(L, sz[tid], fk);
      z[p * DK + tid] = zn;
      part = fq * zn;
    }
    part = warp_sum(part);
    if ((tid & 31) == 0) s_den[tid >> 5] = part;
    __syncthreads();

    float4 vv;
    vv.x = to_f32(sv[4 * c4 + 0]);
    vv.y = to_f32(sv[4 * c4 + 1]);
    vv.z = to_f32(sv[4 * c4 + 2]);
    vv.w = to_f32(sv[4 * c4 + 3]);
    float4 *Sp = reinterpret_cast<float4 *>(S + p * DK * DV);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int j = 0; j < PASSES; ++j) {
      const int r = r0 + j * RPP;
      if (r < DK) {
        const float fk = s_fk[r], fq = s_fq[r];
        float4 t = *reinterpret_cast<const float4 *>(sS + r * DV + 4 * c4);
        t.x = fmaf(L, t.x, fk * vv.x);
        t.y = fmaf(L, t.y, fk * vv.y);
        t.z = fmaf(L, t.z, fk * vv.z);
        t.w = fmaf(L, t.w, fk * vv.w);
        __stcs(&Sp[r * TPR + c4], t);
        acc.x = fmaf(fq, t.x, acc.x);
        acc.y = fmaf(fq, t.y, acc.y);
        acc.z = fmaf(fq, t.z, acc.z);
        acc.w = fmaf(fq, t.w, acc.w);
      }
    }
    *reinterpret_cast<float4 *>(&s_red[r0 * DV + 4 * c4]) = acc;
    __syncthreads();
    // every read of this stage is done: refill it with head i + stages
    if (tid == 0 && i + kDecodeStages < nmine) {
      fence_proxy_async_smem();
      issue(i + kDecodeStages);
    }
    if (tid < DV) {
      float num = 0.f;
#pragma unroll 8
      for (int r = 0; r < RPP; ++r) num += s_red[r * DV + tid];
      float den = 0.f;
#pragma unroll
      for (int w = 0; w < NT / 32; ++w) den += s_den[w];
      out[p * DV + tid] = from_f32<T>(num / (den + eps));
    }
    __syncthreads();
  }
  if (*abort_flag && tid == 0) {
    // drain the copies still in flight (bounded waits)
    for (int j = i; j < nmine && j < i + kDecodeStages; ++j)
      mbar_wait(bar0 + 8 * (j % kDecodeStages), (j / kDecodeStages) & 1);
  }
}

}  // namespace linattn
