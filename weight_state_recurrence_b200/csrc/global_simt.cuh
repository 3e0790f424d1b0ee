// Global (non-causal) form on CUDA cores, fp32 arithmetic.
//   pass 1: KV = sum_n phi(k_n) v_n^T and ksum = sum_n phi(k_n) over the keys
//           that are not padding, split over N across CTAs and accumulated
//           with fp32 atomics into the caller's (zeroed) KV / ksum;
//   pass 2: y_i = phi(q_i)^T KV / (phi(q_i)^T ksum + eps).
// Linear-attention note §3 (after the sum swap) and §6 forward; "Beyond
// self-attention", linear-attention code (here with eps).
// This is the path for fp32 inputs and for sizes the tensor-core kernel does
// not cover.
#pragma once
#include "common.cuh"

namespace linattn {

constexpr int kGlobalTile = 32;     // tokens staged per iteration
constexpr int kGlobalSplit = 512;   // tokens per pass-1 CTA

// kpm: key padding mask [B, N] (nonzero: the key is padding and enters
// neither sum) or NULL; H: heads per sequence (to find a pair's row of kpm).
template <int DK, int DV, typename T>
__global__ void __launch_bounds__(256) global_kv_simt_kernel(const T *__restrict__ k,
                                                             const T *__restrict__ v,
                                                             const uint8_t *__restrict__ kpm,
                                                             float *__restrict__ KV,
                                                             float *__restrict__ ksum, int N,
                                                             int H, bool ident) {
  constexpr int NT = 256, TT = kGlobalTile;
  constexpr int ENT = DK * DV;
  constexpr int PER = (ENT + NT - 1) / NT;
  __shared__ float sK[TT][DK];
  __shared__ float sV[TT][DV];
  const long pair = blockIdx.x;
  const int n0 = blockIdx.y * kGlobalSplit;
  const int n1 = min(N, n0 + kGlobalSplit);
  const int tid = threadIdx.x;
  float acc[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) acc[i] = 0.f;
  float ks = 0.f;
  const uint8_t *mrow = kpm ? kpm + (pair / H) * static_cast<long>(N) : nullptr;
  for (int t0 = n0; t0 < n1; t0 += TT) {
    const int tv = min(TT, n1 - t0);
    __syncthreads();
    for (int i = tid; i < TT * DK; i += NT) {
      const int t = i / DK, a = i % DK;
      const bool live = t < tv && !(mrow && mrow[t0 + t]);
      sK[t][a] = live ? feat_f32(to_f32(k[(pair * N + t0 + t) * DK + a]), ident) : 0.f;
    }
    for (int i = tid; i < TT * DV; i += NT) {
      const int t = i / DV, b = i % DV;
      sV[t][b] = t < tv ? to_f32(v[(pair * N + t0 + t) * DV + b]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int e = tid + i * NT;
      if (e < ENT) {
        const int a = e / DV, b = e % DV;
        float s = acc[i];
        for (int t = 0; t < tv; ++t) s = fmaf(sK[t][a], sV[t][b], s);
        acc[i] = s;
      }
    }
    if (tid < DK)
      for (int t = 0; t < tv; ++t) ks += sK[t][tid];
  }
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int e = tid + i * NT;
    if (e < ENT) atomicAdd(&KV[pair * ENT + e], acc[i]);
  }
  if (tid < DK) atomicAdd(&ksum[pair * DK + tid], ks);
}

template <int DK, int DV, typename T>
__global__ void __launch_bounds__(256) global_out_simt_kernel(const T *__restrict__ q,
                                                              const float *__restrict__ KV,
                                                              const float *__restrict__ ksum,
                                                              float eps, T *__restrict__ out,
                                                              int N, bool ident) {
  constexpr int NT = 256, TT = kGlobalTile;
  extern __shared__ __align__(16) float gsm[];
  float *sKV = gsm;              // [DK][DV]
  float *sks = sKV + DK * DV;    // [DK]
  float *sQ = sks + DK;          // [TT][DK+1]
  float *sden = sQ + TT * (DK + 1);  // [TT]
  const long pair = blockIdx.x;
  const int t0 = blockIdx.y * TT;
  const int tv = min(TT, N - t0);
  const int tid = threadIdx.x;
  for (int i = tid; i < DK * DV; i += NT) sKV[i] = KV[pair * DK * DV + i];
  for (int i = tid; i < DK; i += NT) sks[i] = ksum[pair * DK + i];
  for (int i = tid; i < TT * DK; i += NT) {
    const int t = i / DK, a = i % DK;
    sQ[t * (DK + 1) + a] = t < tv ? feat_f32(to_f32(q[(pair * N + t0 + t) * DK + a]), ident) : 0.f;
  }
  __syncthreads();
  for (int t = tid; t < TT; t += NT) {
    float d = 0.f;
    for (int a = 0; a < DK; ++a) d = fmaf(sQ[t * (DK + 1) + a], sks[a], d);
    sden[t] = d + eps;
  }
  __syncthreads();
  for (int i = tid; i < TT * DV; i += NT) {
    const int t = i / DV, b = i % DV;
    if (t >= tv) continue;
    float num = 0.f;
    for (int a = 0; a < DK; ++a) num = fmaf(sQ[t * (DK + 1) + a], sKV[a * DV + b], num);
    out[(pair * N + t0 + t) * DV + b] = from_f32<T>(num / sden[t]);
  }
}

}  // namespace linattn
