// Single-token decode step: one pass over each head's fp32 state.
//
//   S <- lambda S + phi(k) v^T,  z <- lambda z + phi(k),
//   y  = phi(q)^T S / (phi(q)^T z + eps)
// (fast-weight article §4.1 forward_step and §3.1 constant d x d cache;
//  linear-attention note §5 and §6 forward_autoregressive).
//
// The step is bound by HBM traffic on the state: every head reads and
// writes dk*dv*4 bytes of S.  One CTA of 256 threads owns one head; each
// thread owns a float4 column group of dv and a strided set of rows, issues
// all of its 128-bit loads of S before any use (streaming, evict-first), does
// the rank-1 update and the query read in registers and writes S back with
// streaming stores.  The column sums of phi(q)^T S are combined across rows
// through shared memory; phi(q)^T z is a warp-shuffle reduction.
#pragma once
#include "common.cuh"

namespace linattn {

template <int DK, int DV, typename T>
__global__ void __launch_bounds__(256) decode_step_kernel(
    const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
    const float *__restrict__ lam, float eps, float *__restrict__ S, float *__restrict__ z,
    T *__restrict__ out, int H) {
  constexpr int NT = 256;
  constexpr int TPR = DV / 4;            // threads per state row (one float4 each)
  constexpr int RPP = NT / TPR;          // rows covered by the block in one pass
  constexpr int PASSES = (DK + RPP - 1) / RPP;
  static_assert(DV % 4 == 0 && TPR <= NT, "dv must be a multiple of 4, at most 1024");

  __shared__ float s_fk[DK], s_fq[DK];
  __shared__ __align__(16) float s_v[DV];
  __shared__ __align__(16) float s_red[RPP * DV];
  __shared__ float s_den[NT / 32];

  const long p = blockIdx.x;  // (b, h) pair
  const int h = static_cast<int>(p % H);
  const int tid = threadIdx.x;
  const float L = lam ? lam[h] : 1.f;

  float part = 0.f;
  if (tid < DK) {
    const float fk = phi_f32(to_f32(k[p * DK + tid]));
    const float fq = phi_f32(to_f32(q[p * DK + tid]));
    s_fk[tid] = fk;
    s_fq[tid] = fq;
    const float zn = fmaf(L, z[p * DK + tid], fk);
    z[p * DK + tid] = zn;
    part = fq * zn;
  }
  if (tid < DV) s_v[tid] = to_f32(v[p * DV + tid]);
  part = warp_sum(part);
  if ((tid & 31) == 0) s_den[tid >> 5] = part;
  __syncthreads();

  const int c4 = tid % TPR;
  const int r0 = tid / TPR;
  const float4 v4 = *reinterpret_cast<const float4 *>(&s_v[4 * c4]);
  float4 *Sp = reinterpret_cast<float4 *>(S + p * DK * DV);

  float4 s[PASSES];
#pragma unroll
  for (int i = 0; i < PASSES; ++i) {
    const int r = r0 + i * RPP;
    if (r < DK) s[i] = __ldcs(&Sp[r * TPR + c4]);
  }
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int i = 0; i < PASSES; ++i) {
    const int r = r0 + i * RPP;
    if (r < DK) {
      const float fk = s_fk[r], fq = s_fq[r];
      float4 t = s[i];
      t.x = fmaf(L, t.x, fk * v4.x);
      t.y = fmaf(L, t.y, fk * v4.y);
      t.z = fmaf(L, t.z, fk * v4.z);
      t.w = fmaf(L, t.w, fk * v4.w);
      __stcs(&Sp[r * TPR + c4], t);
      acc.x = fmaf(fq, t.x, acc.x);
      acc.y = fmaf(fq, t.y, acc.y);
      acc.z = fmaf(fq, t.z, acc.z);
      acc.w = fmaf(fq, t.w, acc.w);
    }
  }
  *reinterpret_cast<float4 *>(&s_red[r0 * DV + 4 * c4]) = acc;
  __syncthreads();
  if (tid < DV) {
    float num = 0.f;
#pragma unroll 8
    for (int r = 0; r < RPP; ++r) num += s_red[r * DV + tid];
    float den = 0.f;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) den += s_den[w];
    out[p * DV + tid] = from_f32<T>(num / (den + eps));
  }
}

}  // namespace linattn
