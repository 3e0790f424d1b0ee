// Chunked causal forward on CUDA cores, fp32 arithmetic throughout.
//
// This is the path for fp32 inputs (whose 1e-4 accuracy target rules out
// bf16/tf32 tensor-core operands) and for sizes the tensor-core kernel does
// not cover.  It computes the same chunked form as the tensor-core kernel
// (fast-weight article §3.1 triangular mask, §4.1/§5.2 blockwise
// accumulation) with C = 32 tokens per chunk.  For a chunk starting after
// state (S, z), token t (0-based, Cv valid tokens):
//   A[t][s]  = lambda^(t-s) phi(q_t).phi(k_s)        for s <= t, else 0
//   y_t      = (sum_s A[t][s] v_s + lambda^(t+1) phi(q_t)^T S)
//              / (sum_s A[t][s] + lambda^(t+1) phi(q_t).z + eps)
//   S       <- lambda^Cv S + sum_s lambda^(Cv-1-s) phi(k_s) v_s^T
//   z       <- lambda^Cv z + sum_s lambda^(Cv-1-s) phi(k_s)
// which unrolls the recurrence S_i = lambda S_{i-1} + phi(k_i) v_i^T exactly.
// One CTA owns one (b, h) and a DVS-wide slice of dv; S for the slice lives in
// shared memory for the whole sequence, starting from the caller's state if
// one is given.
#pragma once
#include "common.cuh"

namespace linattn {

constexpr int kSimtChunk = 32;

template <int DK, int DVS>
constexpr int causal_simt_smem_floats() {
  constexpr int C = kSimtChunk;
  return 2 * C * (DK + 1) + C * DVS + C * (C + 1) + DK * DVS + DK + (C + 4) + C;
}

template <int DK, int DVS, typename T>
__global__ void __launch_bounds__(256) causal_simt_kernel(
    const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
    const float *__restrict__ lam, float eps, const float *__restrict__ S_init,
    const float *__restrict__ z_init, T *__restrict__ out, float *__restrict__ S_final,
    float *__restrict__ z_final, int H, int N, int DV, int seg_len,
    const float *__restrict__ S_seg, const float *__restrict__ z_seg, bool ident) {
  constexpr int C = kSimtChunk, NT = 256, QS = DK + 1;
  static_assert(DVS % 4 == 0, "slice must be float4-divisible");
  extern __shared__ __align__(16) float sm[];
  float *sQ = sm;                  // [C][DK+1]  phi(q)
  float *sK = sQ + C * QS;         // [C][DK+1]  phi(k)
  float *sV = sK + C * QS;         // [C][DVS]   v slice (later decay-weighted)
  float *sA = sV + C * DVS;        // [C][C+1]   masked, decayed scores
  float *sS = sA + C * (C + 1);    // [DK][DVS]  state slice
  float *sz = sS + DK * DVS;       // [DK]       normaliser
  float *pw = sz + DK;             // [C+1]      lambda^i
  float *sqz = pw + (C + 4);       // [C]        phi(q_t).z

  const int nslices = DV / DVS;
  const long pair = blockIdx.x / nslices;
  const int j0 = (blockIdx.x % nslices) * DVS;
  const int h = static_cast<int>(pair % H);
  const int tid = threadIdx.x;
  const float L = lam ? lam[h] : 1.f;

  if (tid <= C) pw[tid] = pow_int(L, tid);
  // segment blockIdx.y of gridDim.y covers tokens [n0, n1); with segments its
  // starting state is its slot of (S_seg, z_seg), otherwise the caller's
  // (S_init, z_init) or zero
  const int G = gridDim.y, g = blockIdx.y;
  const int n0 = g * seg_len, n1 = min(N, n0 + seg_len);
  const float *S0 = S_seg ? S_seg + (pair * G + g) * static_cast<long>(DK) * DV : S_init;
  const float *z0 = z_seg ? z_seg + (pair * G + g) * static_cast<long>(DK) : z_init;
  const long s0off = S_seg ? 0 : pair * static_cast<long>(DK) * DV;
  const long z0off = z_seg ? 0 : pair * static_cast<long>(DK);
  for (int i = tid; i < DK * DVS; i += NT)
    sS[i] = S0 ? S0[s0off + (i / DVS) * static_cast<long>(DV) + j0 + i % DVS] : 0.f;
  for (int i = tid; i < DK; i += NT) sz[i] = z0 ? z0[z0off + i] : 0.f;

  const T *qp = q + pair * static_cast<long>(N) * DK;
  const T *kp = k + pair * static_cast<long>(N) * DK;
  const T *vp = v + pair * static_cast<long>(N) * DV;
  T *op = out + pair * static_cast<long>(N) * DV;

  for (int c0 = n0; c0 < n1; c0 += C) {
    const int Cv = min(C, n1 - c0);
    __syncthreads();
    {
      // eight elements per load, every load of the chunk in flight before the
      // first shared-memory store
      constexpr int QI = (C * DK / 8 + NT - 1) / NT, VI = (C * DVS / 8 + NT - 1) / NT;
      float fq[QI][8], fk[QI][8], fv[VI][8];
#pragma unroll
      for (int u = 0; u < QI; ++u) {
        const int i = tid + u * NT, t = i / (DK / 8), a = (i % (DK / 8)) * 8;
#pragma unroll
        for (int e = 0; e < 8; ++e) fq[u][e] = fk[u][e] = 0.f;
        if (i < C * DK / 8 && t < Cv) {
          load8_f32(qp + static_cast<long>(c0 + t) * DK + a, fq[u]);
          load8_f32(kp + static_cast<long>(c0 + t) * DK + a, fk[u]);
        }
      }
#pragma unroll
      for (int u = 0; u < VI; ++u) {
        const int i = tid + u * NT, t = i / (DVS / 8), j = (i % (DVS / 8)) * 8;
#pragma unroll
        for (int e = 0; e < 8; ++e) fv[u][e] = 0.f;
        if (i < C * DVS / 8 && t < Cv) load8_f32(vp + static_cast<long>(c0 + t) * DV + j0 + j, fv[u]);
      }
#pragma unroll
      for (int u = 0; u < QI; ++u) {
        const int i = tid + u * NT, t = i / (DK / 8), a = (i % (DK / 8)) * 8;
        if (i >= C * DK / 8) continue;
        const bool live = t < Cv;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          sQ[t * QS + a + e] = live ? feat_f32(fq[u][e], ident) : 0.f;
          sK[t * QS + a + e] = live ? feat_f32(fk[u][e], ident) : 0.f;
        }
      }
#pragma unroll
      for (int u = 0; u < VI; ++u) {
        const int i = tid + u * NT;
        if (i >= C * DVS / 8) continue;
        *reinterpret_cast<float4 *>(&sV[8 * i]) = make_float4(fv[u][0], fv[u][1], fv[u][2], fv[u][3]);
        *reinterpret_cast<float4 *>(&sV[8 * i + 4]) = make_float4(fv[u][4], fv[u][5], fv[u][6], fv[u][7]);
      }
    }
    __syncthreads();
    // masked decayed scores and phi(q_t).z (z is still the state before the chunk)
    for (int i = tid; i < C * C; i += NT) {
      const int t = i / C, s = i % C;
      float a = 0.f;
      if (s <= t && t < Cv) {
        float d = 0.f;
#pragma unroll 8
        for (int c = 0; c < DK; ++c) d = fmaf(sQ[t * QS + c], sK[s * QS + c], d);
        a = pw[t - s] * d;
      }
      sA[t * (C + 1) + s] = a;
    }
    for (int t = tid; t < C; t += NT) {
      float d = 0.f;
      for (int c = 0; c < DK; ++c) d = fmaf(sQ[t * QS + c], sz[c], d);
      sqz[t] = d;
    }
    __syncthreads();
    // outputs: each thread one token and four columns of the slice
    for (int i = tid; i < C * (DVS / 4); i += NT) {
      const int t = i / (DVS / 4), j = 4 * (i % (DVS / 4));
      if (t >= Cv) continue;
      float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
      float rs = 0.f;
      for (int s = 0; s <= t; ++s) {
        const float a = sA[t * (C + 1) + s];
        const float4 vv = *reinterpret_cast<const float4 *>(&sV[s * DVS + j]);
        num.x = fmaf(a, vv.x, num.x);
        num.y = fmaf(a, vv.y, num.y);
        num.z = fmaf(a, vv.z, num.z);
        num.w = fmaf(a, vv.w, num.w);
        rs += a;
      }
      float4 in = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int c = 0; c < DK; ++c) {
        const float fq = sQ[t * QS + c];
        const float4 ss = *reinterpret_cast<const float4 *>(&sS[c * DVS + j]);
        in.x = fmaf(fq, ss.x, in.x);
        in.y = fmaf(fq, ss.y, in.y);
        in.z = fmaf(fq, ss.z, in.z);
        in.w = fmaf(fq, ss.w, in.w);
      }
      const float g = pw[t + 1];
      const float inv = 1.f / (rs + g * sqz[t] + eps);
      T *o = op + static_cast<long>(c0 + t) * DV + j0 + j;
      o[0] = from_f32<T>(fmaf(g, in.x, num.x) * inv);
      o[1] = from_f32<T>(fmaf(g, in.y, num.y) * inv);
      o[2] = from_f32<T>(fmaf(g, in.z, num.z) * inv);
      o[3] = from_f32<T>(fmaf(g, in.w, num.w) * inv);
    }
    __syncthreads();
    // weight value rows by lambda^(Cv-1-s) for the state update
    for (int i = tid; i < C * DVS; i += NT) {
      const int s = i / DVS;
      sV[i] = s < Cv ? sV[i] * pw[Cv - 1 - s] : 0.f;
    }
    __syncthreads();
    const float gC = pw[Cv];
    for (int i = tid; i < DK * (DVS / 4); i += NT) {
      const int c = i / (DVS / 4), j = 4 * (i % (DVS / 4));
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int s = 0; s < Cv; ++s) {
        const float f = sK[s * QS + c];
        const float4 vv = *reinterpret_cast<const float4 *>(&sV[s * DVS + j]);
        acc.x = fmaf(f, vv.x, acc.x);
        acc.y = fmaf(f, vv.y, acc.y);
        acc.z = fmaf(f, vv.z, acc.z);
        acc.w = fmaf(f, vv.w, acc.w);
      }
      float4 *sp = reinterpret_cast<float4 *>(&sS[c * DVS + j]);
      float4 st = *sp;
      st.x = fmaf(gC, st.x, acc.x);
      st.y = fmaf(gC, st.y, acc.y);
      st.z = fmaf(gC, st.z, acc.z);
      st.w = fmaf(gC, st.w, acc.w);
      *sp = st;
    }
    for (int c = tid; c < DK; c += NT) {
      float a = 0.f;
      for (int s = 0; s < Cv; ++s) a = fmaf(sK[s * QS + c], pw[Cv - 1 - s], a);
      sz[c] = fmaf(gC, sz[c], a);
    }
  }
  __syncthreads();
  if (g != G - 1) return;   // only the last segment ends at the sequence's end
  if (S_final) {
    for (int i = tid; i < DK * DVS; i += NT) {
      const int c = i / DVS, j = i % DVS;
      S_final[(pair * DK + c) * DV + j0 + j] = sS[i];
    }
  }
  if (z_final && j0 == 0) {
    for (int c = tid; c < DK; c += NT) z_final[pair * DK + c] = sz[c];
  }
}

// ------------------------------------------------ segment-parallel form
// For few (b, h) the sequence is cut into G segments of seg_len tokens
// (blockwise accumulation of [FW] §4.1 note and §5.2, one level up: the
// "parallel scan" alternative).  (1) Each segment but the last computes the
// state it would end in from zero, dS_g = sum_{j in g} lambda^(end_g - j)
// phi(k_j) v_j^T and dz_g likewise; (2) one pass per head turns them into the
// starting state of every segment, carry_{g+1} = lambda^(len_g) carry_g + dS_g
// with carry_0 the caller's starting state; (3) the chunked kernel above runs
// all segments at once, each from its carry.  dS_g and carry_g share one slot
// of the workspace ([B*H][G][DK][DV] fp32, then [B*H][G][DK] fp32).

template <int DK, int DVS, typename T>
__global__ void __launch_bounds__(256) causal_seg_state_kernel(
    const T *__restrict__ k, const T *__restrict__ v, const float *__restrict__ lam,
    float *__restrict__ ws_S, float *__restrict__ ws_z, int H, int N, int DV, int seg_len,
    int slots, bool ident) {
  constexpr int C = kSimtChunk, NT = 256, QS = DK + 1;
  constexpr int NR = DK / 16, NCOL = DVS / 16;
  __shared__ float sK[C * QS];      // lambda^(Cv-1-s) phi(k_s)
  __shared__ float sV[C * (DVS + 1)];
  __shared__ float pw[C + 4];
  const int nslices = DV / DVS;
  const long pair = blockIdx.x / nslices;
  const int j0 = (blockIdx.x % nslices) * DVS;
  const int g = blockIdx.y, tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  const float L = lam ? lam[pair % H] : 1.f;
  if (tid < C + 4) pw[tid] = pow_int(L, tid);
  const int n0 = g * seg_len, n1 = min(N, n0 + seg_len);
  const T *kp = k + pair * static_cast<long>(N) * DK;
  const T *vp = v + pair * static_cast<long>(N) * DV;
  float acc[NR][NCOL] = {};
  float zacc = 0.f;                 // thread a < DK: the normaliser's row a
  for (int c0 = n0; c0 < n1; c0 += C) {
    const int Cv = min(C, n1 - c0);
    __syncthreads();
    {
      // eight elements per load, every load of the chunk in flight before the
      // first shared-memory store
      constexpr int KI = (C * DK / 8 + NT - 1) / NT, VI = (C * DVS / 8 + NT - 1) / NT;
      float fk[KI][8], fv[VI][8];
#pragma unroll
      for (int u = 0; u < KI; ++u) {
        const int i = tid + u * NT, t = i / (DK / 8), a = (i % (DK / 8)) * 8;
#pragma unroll
        for (int e = 0; e < 8; ++e) fk[u][e] = 0.f;
        if (i < C * DK / 8 && t < Cv) load8_f32(kp + static_cast<long>(c0 + t) * DK + a, fk[u]);
      }
#pragma unroll
      for (int u = 0; u < VI; ++u) {
        const int i = tid + u * NT, t = i / (DVS / 8), j = (i % (DVS / 8)) * 8;
#pragma unroll
        for (int e = 0; e < 8; ++e) fv[u][e] = 0.f;
        if (i < C * DVS / 8 && t < Cv) load8_f32(vp + static_cast<long>(c0 + t) * DV + j0 + j, fv[u]);
      }
#pragma unroll
      for (int u = 0; u < KI; ++u) {
        const int i = tid + u * NT, t = i / (DK / 8), a = (i % (DK / 8)) * 8;
        if (i >= C * DK / 8) continue;
        const float w = t < Cv ? pw[Cv - 1 - t] : 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) sK[t * QS + a + e] = t < Cv ? w * feat_f32(fk[u][e], ident) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < VI; ++u) {
        const int i = tid + u * NT, t = i / (DVS / 8), j = (i % (DVS / 8)) * 8;
        if (i >= C * DVS / 8) continue;
#pragma unroll
        for (int e = 0; e < 8; ++e) sV[t * (DVS + 1) + j + e] = fv[u][e];
      }
    }
    __syncthreads();
    const float gC = pw[Cv];
#pragma unroll
    for (int r = 0; r < NR; ++r)
#pragma unroll
      for (int m = 0; m < NCOL; ++m) acc[r][m] *= gC;
    for (int t = 0; t < Cv; ++t) {
      float x[NR], y[NCOL];
#pragma unroll
      for (int r = 0; r < NR; ++r) x[r] = sK[t * QS + ty + 16 * r];
#pragma unroll
      for (int m = 0; m < NCOL; ++m) y[m] = sV[t * (DVS + 1) + tx + 16 * m];
#pragma unroll
      for (int r = 0; r < NR; ++r)
#pragma unroll
        for (int m = 0; m < NCOL; ++m) acc[r][m] = fmaf(x[r], y[m], acc[r][m]);
    }
    if (tid < DK) {
      zacc *= gC;
      for (int t = 0; t < Cv; ++t) zacc += sK[t * QS + tid];
    }
  }
  float *Sg = ws_S + (pair * slots + g) * static_cast<long>(DK) * DV;
#pragma unroll
  for (int r = 0; r < NR; ++r)
#pragma unroll
    for (int m = 0; m < NCOL; ++m) Sg[(ty + 16 * r) * static_cast<long>(DV) + j0 + tx + 16 * m] = acc[r][m];
  if (j0 == 0 && tid < DK) ws_z[(pair * slots + g) * static_cast<long>(DK) + tid] = zacc;
}

// carry_0 = (S_init, z_init) or zero; carry_{g+1} = lambda^len_g carry_g + dS_g,
// written over dS_g's slot.  Grid: blockIdx.x is the (b, h) pair, blockIdx.y
// a block of 256 of its DK*DV + DK state elements, one element per thread.
__global__ void __launch_bounds__(256) causal_seg_combine_kernel(
    const float *__restrict__ lam, const float *__restrict__ S_init,
    const float *__restrict__ z_init, float *__restrict__ ws_S, float *__restrict__ ws_z, int H,
    int DK, int DV, long N, int seg_len, int G, bool seg_major) {
  // blockIdx.x: the (b, h) pair; blockIdx.y: a block of 256 of its DK*DV + DK
  // state elements, one per thread.  Each element's G segment values are read
  // eight at a time before any is overwritten, so a thread has eight loads in
  // flight instead of one per step of its scan.
  __shared__ float decay[64];       // lambda^len_g
  const long pair = blockIdx.x;
  const float L = lam ? lam[pair % H] : 1.f;
  for (int gg = threadIdx.x; gg < G; gg += blockDim.x)
    decay[gg] = pow_int(L, static_cast<int>(min(static_cast<long>(seg_len),
                                                 N - static_cast<long>(gg) * seg_len)));
  __syncthreads();
  const long per = static_cast<long>(DK) * DV;
  const long e = static_cast<long>(blockIdx.y) * blockDim.x + threadIdx.x;
  if (e >= per + DK) return;
  const bool isz = e >= per;
  const long ei = isz ? e - per : e;
  const long unit = isz ? DK : per;   // one state's elements
  // [B*H][G] slots (the segmented forward's workspace) or [G][B*H] (segment
  // states gathered from several devices)
  float *base = (isz ? ws_z : ws_S) + (seg_major ? pair : pair * G) * unit;
  const long stride = seg_major ? static_cast<long>(gridDim.x) * unit : unit;
  const float *init = isz ? z_init : S_init;
  float run = init ? init[pair * unit + ei] : 0.f;
  for (int g0 = 0; g0 < G; g0 += 8) {
    float d[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int gg = g0 + j;
      d[j] = gg < G - 1 ? base[gg * stride + ei] : 0.f;
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int gg = g0 + j;
      if (gg < G) {
        base[gg * stride + ei] = run;
        run = fmaf(decay[gg], run, d[j]);
      }
    }
  }
}

}  // namespace linattn
