// Chunked causal forward on the 5th-generation tensor cores, one CTA per
// (head, segment of the sequence) with the head's whole d_v, plus the
// tensor-core state pass that gives every segment after the first its
// starting state.  bf16 operands, fp32 accumulators in TMEM, d_k and d_v in
// {64, 128}.
//
// The method (fast-weight article §2.1/§3.2/§4.2 recurrence; §3.1 triangular
// mask; §4.1 note and §5.2: cut the sequence into blocks, parallel inside a
// block, carried across blocks; the "parallel scan" over segments of §5.2 is
// the split into segments), per chunk of C = 128 tokens, t and s 0-based in
// the chunk, Cv valid tokens, carried state (S, z):
//
//   P    = (phi(Q) phi(K)^T) o M,   M[t][s] = lambda^(t-s) for s <= t, else 0
//   num  = P V + Lq phi(Q) S,       Lq = diag(lambda^(t+1))
//   den  = P 1 + Lq phi(Q) z + eps
//   y    = num / den
//   S   <- lambda^Cv S + (Lk phi(K))^T V,   Lk = diag(lambda^(Cv-1-s))
//   z   <- lambda^Cv z + (Lk phi(K))^T 1
//
// Tensor-core chains per chunk (M = 128, K = 16 per instruction, N = d_v):
//   score   D_A   = phi(Q) phi(K)^T                       TMEM x SMEM
//   carried D_O   = phi(Q) S'        (S' = bf16 state)    TMEM x SMEM
//   state   D_S  += (Lk phi(K))^T V                       SMEM x SMEM (both MN-major)
//   intra   D_O  += P V              (P = bf16 in TMEM)   TMEM x SMEM
// One accumulator takes both halves of the numerator.  phi(Q) is written to
// TMEM by the feature-map warps, so three of the four chains read only their
// B operand from shared memory: an MMA that reads both operands there takes
// shared-memory bandwidth that the feature map needs.  The denominator is
// formed in fp32 on the CUDA cores: the feature-map warps keep z and take
// phi(q_t).z while they transform q; the score epilogue adds the fp32 row sums
// of the masked score tile (the numerator uses the same weights rounded to
// bf16, a relative difference below 2^-9).
//
// Decay.  For lambda >= kFactorMin the decay is factored into the operands
// relative to a frame of R chunks that starts at token n_f: the q row of
// token p is scaled by lambda^(p+1-n_f) and the k row by lambda^(n_f-1-p)
// while the feature map is applied.  The score MMA then yields lambda^(t-s)
// phi(q_t).phi(k_s), the state MMA accumulates S~ = lambda^-(n-n_f) S with
// no decay between chunks, and phi(q') S~ is the carried term itself; the
// state warps only convert S~ to the bf16 operand, and once per frame
// multiply it by lambda^(R C) (frame_chunks bounds the weights).  Smaller
// lambda (down to 0): the score epilogue multiplies by lambda^(t-s), after
// the score MMA has read them the q rows are rescaled by lambda^(t+1) and the
// k rows by lambda^(Cv-1-s), and the state is decayed by lambda^Cv before
// every state MMA.
//
// Warp roles (1024 threads):
//   warp 0      TMA producer of the q and k tiles
//   warp 1      TMEM owner, the single MMA-issuing thread
//   warp 2      TMA producer of the v tiles
//   warps 4-7   score epilogue: D_A -> mask (and decay) -> bf16 P in TMEM, row sums
//   warps 8-11  output: y = D_O / den -> global memory (D_O single-buffered:
//               the next carried product waits until it is drained)
//   warps 12-15 state: D_S -> bf16 operand S' (and the decay or renormalisation of D_S)
//   warps 16-31 feature map (packed bf16x2): phi(q) into TMEM, phi(k) in place,
//               phi(q).z, z update
// Every wait is bounded (sm100.cuh); a wait that runs out records an error
// flag and every role leaves its loop.
#pragma once
#include "common.cuh"
#include "sm100.cuh"
#include "causal_tc.cuh"

namespace linattn {
namespace stc {

using tc::mul_bf16x2;
using tc::pack_bf16;
using tc::phi_bf16x2;

constexpr int C = 128;
constexpr int NT = 1024;
constexpr int kPhiThreads = 512;
constexpr int kBarPhi = 1, kBarP = 2, kBarOut = 3, kBarState = 4;   // named barriers
// The thread of each multi-warp role that polls its mbarriers (the others wait
// at the role's named barrier), placed so that the four schedulers of the SM
// (warp % 4) each carry about the same number of polling warps: TMA q 0,
// MMA 1, TMA v 2, TMA k 3, score epilogue warp 4, feature map warp 17,
// state warp 14, output warp 11.
constexpr int kPollPhi = 32, kPollState = 64, kPollOut = 96;
constexpr float kFactorMin = 0.7f;

constexpr uint32_t kPanel = 16384;              // 128 rows x 128 bytes (64 bf16)
constexpr uint32_t kOffQ = 0;                   // per stage: q, 2 panels of d_k
constexpr uint32_t kOffK = 2 * kPanel;          //            k, 2 panels of d_k
constexpr uint32_t kOffV = 4 * kPanel;          //            v, 2 panels of d_v
constexpr uint32_t kStage = 6 * kPanel;         // 96 KB
constexpr uint32_t kOffSop = 2 * kStage;        // bf16 state operand: rows d_k, 2 panels of d_v
constexpr uint32_t kOffMisc = kOffSop + 2 * kPanel;
constexpr uint32_t kMiscTmem = 256, kMiscAbort = 260, kMiscRoleFail = 272;
constexpr uint32_t kMiscPw = 320;               // lambda^i, i = 0..C        (129 floats)
constexpr uint32_t kMiscZ = 848;                // z, fp32                   (128 floats)
constexpr uint32_t kMiscDen = 1360;             // den[3][128]: phi(q).z + row sum of P
constexpr int kDenBufs = 3;
constexpr uint32_t kMiscBytes = kMiscDen + kDenBufs * 128 * 4;
constexpr uint32_t kSmemBytes = kOffMisc + kMiscBytes;
static_assert(kSmemBytes <= 232448, "exceeds the per-CTA shared memory of sm_100");

enum Bar {
  kFullQ0 = 0, kFullQ1, kFullK0, kFullK1, kFullV0, kFullV1, kFreeK0, kFreeK1, kFreeV0, kFreeV1,
  kPhi0, kPhi1, kScore, kRescale, kState, kReadout, kPDone, kO, kOut, kSop,
  kQFree0, kQFree1,   // the score epilogue has read the phi(q).z parts left in q tile s
  // den buffer b (chunk c uses b = c % 3): phi(q).z written, row sums added, read by the output
  kDenQz0, kDenQz1, kDenQz2, kDenRs0, kDenRs1, kDenRs2, kDenFree0, kDenFree1, kDenFree2,
  kFinal, kNumBars
};
static_assert(kNumBars * 8 <= 256, "barrier area overflow");

// tensor memory columns (32-bit, lane = row)
constexpr uint32_t kTmS = 0;     // state D_S, lane = d_k row
constexpr uint32_t kTmA = 128;   // score D_A; P (bf16 pairs) overwrites its first 64 columns
constexpr uint32_t kTmO = 256;   // output accumulator D_O
constexpr uint32_t kTmQ = 384;   // phi(Q') as bf16 pairs, 64 columns per stage (A of score, carried)
constexpr uint32_t kTmCols = 512;

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Sums of 8 values over the 32 lanes of a warp in 9 shuffles: each round
// keeps half of the values and trades the other half with the partner lane.
// Lane L ends with the full sum of value ((L >> 4) & 1) * 4 + ((L >> 3) & 1) * 2
// + ((L >> 2) & 1); lanes that differ only in bits 0-1 hold the same sum.
__device__ __forceinline__ float warp_sum8_transposed(const float (&v)[8], int lane) {
  float a[4], b[2];
  const bool h16 = lane & 16, h8 = lane & 8, h4 = lane & 4;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float send = h16 ? v[i] : v[4 + i];
    a[i] = (h16 ? v[4 + i] : v[i]) + __shfl_xor_sync(0xffffffffu, send, 16);
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const float send = h8 ? a[i] : a[2 + i];
    b[i] = (h8 ? a[2 + i] : a[i]) + __shfl_xor_sync(0xffffffffu, send, 8);
  }
  const float send = h4 ? b[0] : b[1];
  float c = (h4 ? b[1] : b[0]) + __shfl_xor_sync(0xffffffffu, send, 4);
  c += __shfl_xor_sync(0xffffffffu, c, 2);
  c += __shfl_xor_sync(0xffffffffu, c, 1);
  return c;
}
__device__ __forceinline__ int warp_sum8_index(int lane) {
  return ((lane >> 4) & 1) * 4 + ((lane >> 3) & 1) * 2 + ((lane >> 2) & 1);
}

// byte offset of 16-byte chunk j (0..15) of row `row` in a 2-panel K-major tile
__device__ __forceinline__ uint32_t chunk_off(uint32_t row, uint32_t j) {
  return (j >> 3) * kPanel + sw128_offset(row, (j & 7) * 16);
}

// Chunks per frame of the factored decay.  Inside a frame that starts at
// token n_f, the TMEM state is S~ = lambda^-(n - n_f) S (n = tokens seen), the
// k row of token p carries lambda^(n_f - 1 - p) and the q row lambda^(p + 1 -
// n_f), so the state MMA accumulates onto S~ with no decay between chunks
// and the carried term phi(q') S~ is already lambda^(t+1) phi(q) S.  The
// weights stay within 2^+-64 (one chunk at lambda = kFactorMin reaches
// 2^66), so the frame spans at most 64 / (C log2(1/lambda)) chunks; at its end
// the state is multiplied by lambda^(R C) once (a renormalisation).
__device__ __forceinline__ int frame_chunks(float L) {
  if (L >= 1.f) return 1 << 30;
  const float f = 64.f / (static_cast<float>(C) * -log2f(L));
  return f >= static_cast<float>(1 << 20) ? (1 << 20) : max(1, static_cast<int>(f));
}

template <int DKP, int DVP>
__global__ void __launch_bounds__(NT, 1)
    causal_seg_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                         const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const float *__restrict__ lam,
                         float eps, const float *__restrict__ S_init,
                         const float *__restrict__ z_init, const float *__restrict__ ws_S,
                         const float *__restrict__ ws_z, __nv_bfloat16 *__restrict__ out,
                         float *__restrict__ S_final, float *__restrict__ z_final, int H, int N,
                         int seg_len, int G, bool ident) {
  constexpr int DK = 64 * DKP, DV = 64 * DVP;
  constexpr int KCH = 8 * DKP;                  // 16-byte chunks per q/k row
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *sm = smem_raw;
  const uint32_t sb = smem_u32(sm);
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  if (sb & 1023u) {
    if (tid == 0) atomicOr(&g_status, kStatusWaitTimeout);
    return;
  }
  // segment-major: the first segments' CTAs come first, so they start
  // while the state pass of the previous launch is still running
  const long BH = gridDim.x / G;
  const int g = static_cast<int>(blockIdx.x / BH);
  const long pair = blockIdx.x % BH;
  const int h = static_cast<int>(pair % H);
  const float L = lam ? lam[h] : 1.f;
  const int n0 = g * seg_len;
  const int n1 = min(N, n0 + seg_len);
  const int nchunks = (n1 - n0 + C - 1) / C;
  const int Ct = (n1 - n0) - (nchunks - 1) * C;   // valid tokens of the last chunk
  const bool last_seg = g == G - 1;
  // this head's starting state: the caller's (S_init, first segment) or the
  // carry into segment g, summed here from the states of segments 0..g-1
  // that the state pass left in slots pair G + j of the workspace:
  //   S0_g = sum_j lambda^((g-1-j) len) dS_j + lambda^(g len) S_init
  // (every segment before g holds len tokens).  Those CTAs wait for the
  // state pass, which they may overlap when launched as its dependent.
  const float *Sin = S_init ? S_init + pair * DK * static_cast<long>(DV) : nullptr;
  const float *zin = z_init ? z_init + pair * static_cast<long>(DK) : nullptr;
  const bool has_init = g > 0 || Sin != nullptr;
  if (g > 0) grid_dependency_wait();
  // four consecutive elements e..e+3 of the starting S (unit DK DV) or z
  // (unit DK): the newest segment first, each older one lambda^len further back
  const float Llen = g > 0 ? pow_int(L, seg_len) : 1.f;
  auto carry4 = [&](const float *init, const float *slots, long unit, long e) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float f = 1.f;
    for (int j = g - 1; j >= 0; --j) {
      const float4 v = *reinterpret_cast<const float4 *>(slots + (pair * G + j) * unit + e);
      acc = make_float4(fmaf(f, v.x, acc.x), fmaf(f, v.y, acc.y), fmaf(f, v.z, acc.z),
                        fmaf(f, v.w, acc.w));
      f *= Llen;
    }
    if (init) {
      const float4 v = *reinterpret_cast<const float4 *>(init + e);
      acc = make_float4(fmaf(f, v.x, acc.x), fmaf(f, v.y, acc.y), fmaf(f, v.z, acc.z),
                        fmaf(f, v.w, acc.w));
    }
    return acc;
  };
  const bool factored = L >= kFactorMin;
  // factored decay keeps the state in a frame of R chunks (see frame_chunks)
  const int R = factored ? frame_chunks(L) : 1;

  uint8_t *misc = sm + kOffMisc;
  auto bar = [&](int i) { return sb + kOffMisc + 8u * static_cast<uint32_t>(i); };
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(misc + kMiscTmem);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(misc + kMiscAbort);
  volatile int *role_fail = reinterpret_cast<volatile int *>(misc + kMiscRoleFail);
  float *pw = reinterpret_cast<float *>(misc + kMiscPw);
  float *zs = reinterpret_cast<float *>(misc + kMiscZ);
  float *den = reinterpret_cast<float *>(misc + kMiscDen);
  auto Cv_of = [&](int c) { return c == nchunks - 1 ? Ct : C; };

  // ------------------------------------------------------------ set-up
  if (tid == 0) {
    for (int i = 0; i < kNumBars; ++i) mbar_init(bar(i), 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (tid < 4) role_fail[tid] = 0;
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmCols);
    tmem_relinquish();
  }
  if (tid <= C) pw[tid] = pow_int(L, tid);
  if (tid < DK / 4) {
    const float4 z4 = g > 0 ? carry4(zin, ws_z, DK, 4 * tid)
                            : (zin ? reinterpret_cast<const float4 *>(zin)[tid]
                                   : make_float4(0.f, 0.f, 0.f, 0.f));
    reinterpret_cast<float4 *>(zs)[tid] = z4;
  } else if (tid < 32) {
    reinterpret_cast<float4 *>(zs)[tid] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  if (DKP == 1) {
    // the second d_k panel of the q and k tiles stays zero (the state MMA
    // reads it as rows 64-127 of phi(K)^T; the other chains never do)
    for (uint32_t o = tid * 16u; o < 4 * kPanel; o += NT * 16u) {
      const uint32_t st = (o / (2 * kPanel)) * kStage, w = o % (2 * kPanel);
      *reinterpret_cast<uint4 *>(sm + st + (w < kPanel ? kOffQ : kOffK - kPanel) + kPanel + w) =
          make_uint4(0, 0, 0, 0);
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  auto fail = [&]() { *abort_flag = 1; };

  // Starting state, written by every warp (warp w: TMEM lane quarter w % 4,
  // d_v slice w / 4 of DV / 8 columns), so that the carry summed from the
  // state pass's slots costs a few loads per thread: operand S' = S0;
  // explicit decay: D_S = lambda^Cv0 S0 (the state MMA adds chunk 0 onto the
  // decayed state); factored: D_S = S0, the first frame starting at the
  // segment's first token.  Rows d_k..127 of D_S are zero.
  if (has_init && nchunks > 0) {
    constexpr int SC = DV / 8;                  // 16 or 8 columns
    const int r = (warp & 3) * 32 + lane;       // d_k row, TMEM lane
    const int c0 = (warp >> 2) * SC;
    const bool live = r < DK;
    const float g0 = factored ? 1.f : pw[Cv_of(0)];
    uint32_t v[SC], sv[SC];
#pragma unroll
    for (int i = 0; i < SC / 4; ++i) {
      float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
      if (live) {
        const long e = static_cast<long>(r) * DV + c0 + 4 * i;
        f = g == 0 ? *reinterpret_cast<const float4 *>(Sin + e)
                   : carry4(Sin, ws_S, static_cast<long>(DK) * DV, e);
      }
      v[4 * i] = __float_as_uint(f.x);
      v[4 * i + 1] = __float_as_uint(f.y);
      v[4 * i + 2] = __float_as_uint(f.z);
      v[4 * i + 3] = __float_as_uint(f.w);
    }
#pragma unroll
    for (int i = 0; i < SC; ++i) sv[i] = __float_as_uint(__uint_as_float(v[i]) * g0);
    const uint32_t ta = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16) + kTmS + c0;
    if constexpr (SC == 16) tmem_st_32x32b_x16(ta, sv);
    else tmem_st_32x32b_x8(ta, sv);
    uint32_t pk[SC / 2];
#pragma unroll
    for (int i = 0; i < SC / 2; ++i)
      pk[i] = pack_bf16(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
#pragma unroll
    for (int i = 0; i < SC / 8; ++i)
      *reinterpret_cast<uint4 *>(sm + kOffSop + (c0 >> 6) * kPanel +
                                 sw128_offset(r, (c0 & 63) * 2 + i * 16)) =
          make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
    tmem_wait_st();
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  if (warp == 0 || warp == 2 || warp == 3) {
    // ------------------------------------------- TMA producers: q, v, k
    // k is read by the score and state products, v by the state and P V
    // products.  The q tile is read only by the feature map, but loading
    // q(c + 2) lets the feature map overwrite phi(Q') of stage s in TMEM, so
    // the q ring also waits for the MMAs of chunk c to be done with it (the
    // k ring's release) and for the score epilogue to have taken the
    // phi(q).z parts left in the tile.
    if (lane == 0 && nchunks > 0) {
      const int which = warp == 0 ? 0 : (warp == 3 ? 1 : 2);
      const CUtensorMap *map = which == 0 ? &tm_q : (which == 1 ? &tm_k : &tm_v);
      const uint32_t off = which == 0 ? kOffQ : (which == 1 ? kOffK : kOffV);
      const int np = which == 2 ? DVP : DKP;
      const int full0 = which == 0 ? kFullQ0 : (which == 1 ? kFullK0 : kFullV0);
      const int free0 = which == 0 ? kQFree0 : (which == 1 ? kFreeK0 : kFreeV0);
      int issued = 0;
      for (int c = 0; c < nchunks && !*abort_flag; ++c) {
        const int s = c & 1;
        // the stage is needed a chunk from now: wait without taking issue slots
        if (c >= 2 && (!mbar_wait_backoff(bar(free0 + s), ((c - 2) >> 1) & 1) ||
                       (which == 0 && !mbar_wait_backoff(bar(kFreeK0 + s), ((c - 2) >> 1) & 1)))) {
          fail();
          break;
        }
        const int y = n0 + c * C;
        const uint32_t b = bar(full0 + s);
        mbar_arrive_expect_tx(b, np * kPanel);
        for (int p = 0; p < np; ++p)
          tma_load_3d(sb + s * kStage + off + p * kPanel, map, b, 64 * p, y,
                      static_cast<int>(pair));
        if (c + 2 < nchunks)
          for (int p = 0; p < np; ++p)
            tma_prefetch_l2_3d(map, 64 * p, y + 2 * C, static_cast<int>(pair));
        issued = c + 1;
      }
      if (*abort_flag) {
        // let the copies this thread started land before the CTA exits
        for (int c = issued - 2 < 0 ? 0 : issued - 2; c < issued; ++c)
          mbar_wait(bar(full0 + (c & 1)), (c >> 1) & 1);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idA = idesc_bf16(128, 128, 0, 0);    // K-major x K-major
      constexpr uint32_t idQS = idesc_bf16(128, DV, 0, 1);    // K-major x MN-major
      constexpr uint32_t idS = idesc_bf16(128, DV, 1, 1);     // MN-major x MN-major
      // descriptors of every operand tile, per stage; a K step adds its byte
      // offset >> 4 to the start-address field (tiles stay below 256 KB, so
      // the 14-bit field never carries)
      const uint64_t dK = sdesc_sw128(sb + kOffK, 16, 1024);
      const uint64_t dKmn = sdesc_sw128(sb + kOffK, kPanel, 1024);
      const uint64_t dV = sdesc_sw128(sb + kOffV, kPanel, 1024);
      const uint64_t dSop = sdesc_sw128(sb + kOffSop, kPanel, 1024);
      auto kofs = [](int ks) -> uint64_t { return ((ks >> 2) * kPanel + (ks & 3) * 32) >> 4; };
      bool ok = true;
      for (int c = 0; ok && c < nchunks; ++c) {
        const int s = c & 1;
        if (*abort_flag) break;
        // score: D_A = phi(Q') phi(K')^T, phi(Q') from TMEM (the previous
        // chunk's P V, issued before, has read D_A: the chains run in issue order)
        if (!mbar_wait(bar(kPhi0 + s), (c >> 1) & 1)) { ok = false; break; }
        tc_fence_after();
        const uint64_t so = static_cast<uint64_t>(s) * (kStage >> 4);   // stage offset
        const uint64_t k0 = dK + so, kmn0 = dKmn + so, v0 = dV + so;
        const uint32_t qa = tmem + kTmQ + s * 64;
#pragma unroll
        for (int ks = 0; ks < 4 * DKP; ++ks)
          umma_bf16_ts(tmem + kTmA, qa + ks * 8, k0 + kofs(ks), idA, ks > 0);
        umma_commit(bar(kScore));
        // explicit decay: the q and k rows are rescaled once the score MMA has read them
        if (!factored && !mbar_wait(bar(kRescale), c & 1)) { ok = false; break; }
        // carried: D_O = phi(Q') S'  (state before this chunk; the previous
        // chunk's output has drained D_O)
        if (!mbar_wait(bar(kSop), c & 1) || (c >= 1 && !mbar_wait(bar(kOut), (c - 1) & 1))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t dO = tmem + kTmO;
        const bool carried = c > 0 || has_init;
        if (carried) {
#pragma unroll
          for (int ks = 0; ks < 4 * DKP; ++ks)
            umma_bf16_ts(dO, qa + ks * 8, dSop + ks * (2048 >> 4), idQS, ks > 0);
        }
        // state: D_S += (Lk phi(K))^T V
        if (!mbar_wait(bar(kReadout), c & 1) || !mbar_wait(bar(kFullV0 + s), (c >> 1) & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < C / 16; ++ks)
          umma_bf16(tmem + kTmS, kmn0 + ks * (2048 >> 4), v0 + ks * (2048 >> 4), idS,
                    (carried || ks > 0) ? 1u : 0u);
        umma_commit(bar(kState));
        umma_commit(bar(kFreeK0 + s));    // k tile and phi(Q') of this chunk fully read
        // intra: D_O += P V
        if (!mbar_wait(bar(kPDone), c & 1)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < C / 16; ++ks)
          umma_bf16_ts(dO, tmem + kTmA + ks * 8, v0 + ks * (2048 >> 4), idQS,
                       (carried || ks > 0) ? 1u : 0u);
        umma_commit(bar(kO));
        umma_commit(bar(kFreeV0 + s));
      }
      if (!ok) fail();
      umma_commit(bar(kFinal));
      mbar_wait(bar(kFinal), 0);
    }
    __syncwarp();
  } else if (warp >= 4 && warp < 8) {
    // --------------------------------------- score epilogue: P into TMEM
    const int wq = warp - 4;
    const int t = wq * 32 + lane;
    const uint32_t lf = static_cast<uint32_t>(wq * 32) << 16;
    volatile int &rf = role_fail[0];
    for (int c = 0; c < nchunks; ++c) {
      const int s = c & 1;
      // kDenQz orders the feature-map warps' phi(q).z before this role's
      // update of the chunk's den buffer.  One thread polls; the others wait
      // at the named barrier, which takes no issue slots.
      if (t == 0 && (*abort_flag || !mbar_wait(bar(kScore), c & 1) ||
                     !mbar_wait(bar(kDenQz0 + c % kDenBufs), (c / kDenBufs) & 1) ||
                     (c >= kDenBufs && !mbar_wait(bar(kDenFree0 + c % kDenBufs),
                                                  ((c - kDenBufs) / kDenBufs) & 1)))) {
        rf = 1;
        fail();
      }
      named_bar_sync(kBarP, 128);
      tc_fence_after();
      float rs = 0.f;
      float2 rs2 = make_float2(0.f, 0.f);   // the row sum, even and odd keys
      if (!rf) {
        // phi(q').z of row t: the feature-map warps left one part per column
        // block in q tile s, summed here in a fixed order
        const uint8_t *qt = sm + (c & 1) * kStage + kOffQ;
#pragma unroll
        for (int cb = 0; cb < 4; ++cb)
          rs += *reinterpret_cast<const float *>(qt + chunk_off(t, cb * (2 * DKP)));
        // blocks of 32 keys, one load each; only blocks 0..wq hold s <= t
#pragma unroll 1
        for (int bk = 0; bk < 4; ++bk) {
          uint32_t pk[16];
          if (bk <= wq) {
            uint32_t r[32];
            tmem_ld_32x32b_x32(tmem + lf + kTmA + bk * 32, r);
            tmem_wait_ld();
            const int s0 = bk * 32;
            if (factored && bk < wq) {
              // below the diagonal block: every key s <= t, no mask
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const float a = __uint_as_float(r[2 * i]), b = __uint_as_float(r[2 * i + 1]);
                pk[i] = pack_bf16(a, b);
                rs2 = fadd2(rs2, make_float2(a, b));
              }
            } else {
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const int s_a = s0 + 2 * i, s_b = s_a + 1;
                float a = s_a <= t ? __uint_as_float(r[2 * i]) : 0.f;
                float b = s_b <= t ? __uint_as_float(r[2 * i + 1]) : 0.f;
                if (!factored) {
                  a *= s_a <= t ? pw[t - s_a] : 0.f;
                  b *= s_b <= t ? pw[t - s_b] : 0.f;
                }
                pk[i] = pack_bf16(a, b);
                rs2 = fadd2(rs2, make_float2(a, b));
              }
            }
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) pk[i] = 0u;
          }
          // bf16 pairs of keys 32 bk .. 32 bk + 31 into columns 16 bk .. 16 bk + 15,
          // which the loads of this or an earlier block have already read
          tmem_st_32x32b_x16(tmem + lf + kTmA + bk * 16, pk);
        }
        tmem_wait_st();
        den[(c % kDenBufs) * 128 + t] = rs + (rs2.x + rs2.y);
      }
      tc_fence_before();
      named_bar_sync(kBarP, 128);
      if (rf) break;
      if (t == 0) {
        mbar_arrive(bar(kPDone));
        mbar_arrive(bar(kDenRs0 + c % kDenBufs));
        mbar_arrive(bar(kQFree0 + (c & 1)));
      }
    }
  } else if (warp >= 8 && warp < 12) {
    // ---------------------------------------------------------- output y
    const int wq = warp - 8;
    const int t = wq * 32 + lane;
    const uint32_t lf = static_cast<uint32_t>(wq * 32) << 16;
    volatile int &rf = role_fail[1];
    // rows are 128 or 256 bytes, so 32-byte stores need only the base aligned
    const bool out32 = (reinterpret_cast<uintptr_t>(out) & 31u) == 0;
    for (int c = 0; c < nchunks; ++c) {
      if (t == kPollOut && (*abort_flag || !mbar_wait(bar(kO), c & 1) ||
                     !mbar_wait(bar(kDenRs0 + c % kDenBufs), (c / kDenBufs) & 1))) {
        rf = 1;
        fail();
      }
      named_bar_sync(kBarOut, 128);
      tc_fence_after();
      if (!rf) {
        const float inv = 1.f / (den[(c % kDenBufs) * 128 + t] + eps);
        const bool live = t < Cv_of(c);
        uint4 *dst = reinterpret_cast<uint4 *>(
            out + (pair * N + n0 + static_cast<long>(c) * C + (live ? t : 0)) * DV);
#pragma unroll 1
        for (int blk = 0; blk < DV / 32; ++blk) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(tmem + lf + kTmO + blk * 32, r);
          tmem_wait_ld();
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float2 y2 = fmul2(
                make_float2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1])),
                make_float2(inv, inv));
            pk[i] = pack_bf16(y2.x, y2.y);
          }
          if (live) {
            if (out32) {
              st_global_na_v8(dst + blk * 4, pk);
              st_global_na_v8(dst + blk * 4 + 2, pk + 8);
            } else {
#pragma unroll
              for (int i = 0; i < 4; ++i) st_global_na_v4(dst + blk * 4 + i, pk + 4 * i);
            }
          }
        }
      }
      tc_fence_before();
      named_bar_sync(kBarOut, 128);
      if (rf) break;
      if (t == kPollOut) {
        mbar_arrive(bar(kOut));
        mbar_arrive(bar(kDenFree0 + c % kDenBufs));
      }
    }
  } else if (warp >= 12 && warp < 16) {
    // ------------------------------------- state: operand S' and decay
    const int wq = warp - 12;
    const int r = wq * 32 + lane;             // d_k row
    const bool live = r < DK;
    const uint32_t lf = static_cast<uint32_t>(wq * 32) << 16;
    volatile int &rf = role_fail[2];
    // bf16 row of the MN-major operand (row = d_k, 64 d_v per panel)
    // 16 columns (block blk) of this d_k row as bf16 into the operand
    auto put_op = [&](int blk, const uint32_t (&v16)[16], float f) {
      uint32_t pk[8];
      if (f == 1.f) {   // no renormalisation at this chunk: convert only
#pragma unroll
        for (int i = 0; i < 8; ++i)
          pk[i] = pack_bf16(__uint_as_float(v16[2 * i]), __uint_as_float(v16[2 * i + 1]));
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float2 y2 = fmul2(
              make_float2(__uint_as_float(v16[2 * i]), __uint_as_float(v16[2 * i + 1])),
              make_float2(f, f));
          pk[i] = pack_bf16(y2.x, y2.y);
        }
      }
      const uint32_t col = blk * 16;     // first d_v column of this block
#pragma unroll
      for (int i = 0; i < 2; ++i)
        *reinterpret_cast<uint4 *>(sm + kOffSop + (col >> 6) * kPanel +
                                   sw128_offset(r, (col & 63) * 2 + i * 16)) =
            make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
    };
    // the starting state (D_S and S') was written by every warp before the roles began
    fence_proxy_async_smem();
    tc_fence_before();
    named_bar_sync(kBarState, 128);
    if (r == kPollState) {
      mbar_arrive(bar(kSop));
      mbar_arrive(bar(kReadout));
    }
    // lambda^(R C): the renormalisation at the end of a frame (factored)
    const float gR = factored && R < nchunks ? pow_int(L, R * C) : 1.f;
    for (int c = 0; c < nchunks; ++c) {
      const bool last = c == nchunks - 1;
      if (r == kPollState && (*abort_flag || !mbar_wait(bar(kState), c & 1))) {
        rf = 1;
        fail();
      }
      named_bar_sync(kBarState, 128);
      tc_fence_after();
      if (!rf && last && last_seg && S_final) {
        // factored: S = lambda^(tokens since the frame start) S~
        const float fin = factored ? pow_int(pw[C], c % R) * pw[Cv_of(c)] : 1.f;
#pragma unroll 1
        for (int blk = 0; blk < DV / 16; ++blk) {
          uint32_t sv[16];
          tmem_ld_32x32b_x16(tmem + lf + kTmS + blk * 16, sv);   // warp-wide load
          tmem_wait_ld();
          if (live) {
            float4 *dst = reinterpret_cast<float4 *>(S_final + (pair * DK + r) * DV) + blk * 4;
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[i] = make_float4(__uint_as_float(sv[4 * i]) * fin,
                                   __uint_as_float(sv[4 * i + 1]) * fin,
                                   __uint_as_float(sv[4 * i + 2]) * fin,
                                   __uint_as_float(sv[4 * i + 3]) * fin);
          }
        }
      }
      // explicit decay: D_S <- lambda^Cv(next) D_S before every state MMA, the
      // operand unscaled; factored: only at the end of a frame, operand and
      // D_S both renormalised
      const bool decay = !last && (!factored || (c + 1) % R == 0);
      const float gd = factored ? gR : (last ? 1.f : pw[Cv_of(c + 1)]);
      const float fop = factored && decay ? gR : 1.f;
      if (!rf && !last) {
        // (1) the bf16 operand of the next chunk's carried product
#pragma unroll 1
        for (int blk = 0; blk < DV / 16; ++blk) {
          uint32_t sv[16];
          tmem_ld_32x32b_x16(tmem + lf + kTmS + blk * 16, sv);
          tmem_wait_ld();
          put_op(blk, sv, fop);
        }
      }
      fence_proxy_async_smem();
      if (decay) {
        named_bar_sync(kBarState, 128);
        if (rf) break;
        if (r == kPollState) mbar_arrive(bar(kSop));
        if (!rf) {
          // (2) D_S <- gd D_S, before the next state MMA accumulates onto it
#pragma unroll 1
          for (int blk = 0; blk < DV / 16; ++blk) {
            uint32_t sv[16];
            tmem_ld_32x32b_x16(tmem + lf + kTmS + blk * 16, sv);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) sv[i] = __float_as_uint(__uint_as_float(sv[i]) * gd);
            tmem_st_32x32b_x16(tmem + lf + kTmS + blk * 16, sv);
          }
          tmem_wait_st();
        }
        tc_fence_before();
        named_bar_sync(kBarState, 128);
        if (rf) break;
        if (r == kPollState) mbar_arrive(bar(kReadout));
      } else {
        tc_fence_before();
        named_bar_sync(kBarState, 128);
        if (rf) break;
        if (r == kPollState && !last) {
          mbar_arrive(bar(kSop));
          mbar_arrive(bar(kReadout));
        }
      }
    }
  } else if (warp >= 16) {
    // -------------------------------------------------------- feature map
    const int tt = tid - 512;                 // 0..511
    volatile int &rf = role_fail[3];
    auto check = [&](bool ok_wait) {
      if (!ok_wait || *abort_flag) {
        rf = 1;
        fail();
      }
    };
    const int fw = tt >> 5;                   // feature-map warp 0..15
    // q: a thread owns row tq = 32 (warp % 4) + lane, its TMEM lane, and
    // column block cb = fw / 4 (d_k / 4 columns); phi(q') goes to TMEM as the A
    // operand of the score and carried products, and the block's part of
    // phi(q').z is added to the chunk's den
    constexpr int QCH = KCH / 4;              // 16-byte chunks per thread (4 or 2)
    const int tq = (warp & 3) * 32 + lane, cb = fw >> 2;
    const uint32_t lfq = static_cast<uint32_t>((warp & 3) * 32) << 16;
    auto tq_col = [&](int s) { return tmem + lfq + kTmQ + s * 64 + cb * 4 * QCH; };
    // k: a warp owns one column group of 8 columns over all 128 rows, so the
    // column sums of z need no atomics; with d_k = 64 (8 groups) only the
    // first 8 warps take k
    constexpr int NCG = KCH;                  // 16 or 8 column groups
    constexpr int RPL = 128 / 32;             // rows per lane
    const bool kwarp = fw < NCG;
    const int cg = fw;
    float ztot = 0.f;                         // this lane's share of the column sums
    const int zcol = cg * 8 + warp_sum8_index(lane);
    const bool zowner = kwarp && (lane & 3) == 0;
    // factored: Eq = lambda^(tokens from the frame start to this chunk) and
    // Fk = lambda^-(those tokens + C), both stepped by one factor per chunk
    // (no division on the chunk's path; the product Eq Fk lambda^C stays
    // within ~1e-5 of 1 over a frame, far below the bf16 rounding of the
    // operands); explicit: unused
    float Eq = 1.f;
    const float ipwC = factored ? 1.f / pw[C] : 1.f;
    float Fk = ipwC;
    const float gR = factored && R < nchunks ? pow_int(L, R * C) : 1.f;
    for (int c = 0; c < nchunks; ++c) {
      const int s = c & 1;
      const int Cv = Cv_of(c);
      uint8_t *st = sm + s * kStage;
      const bool frame_start = c % R == 0;
      if (factored) {
        Eq = frame_start ? 1.f : Eq * pw[C];
        Fk = frame_start ? ipwC : Fk * ipwC;
      }
      // the previous chunk's column sums: explicit z_{c-1} = lambda^Cv z_{c-2} + sums;
      // factored z~ += sums, renormalised with the state when a frame starts
      if (c > 0 && zowner)
        zs[zcol] = factored ? (frame_start ? gR : 1.f) * (zs[zcol] + ztot)
                            : pw[Cv_of(c - 1)] * zs[zcol] + ztot;
      if (tt == kPollPhi) check(mbar_wait(bar(kFullQ0 + s), (c >> 1) & 1));
      named_bar_sync(kBarPhi, kPhiThreads);
      if (rf) break;
      // (1) q rows: feature map, decay scale, phi(q).z_{c-1}
      {
        float fq;
        if (tq >= Cv) fq = 0.f;
        else fq = factored ? Eq * pw[tq + 1] : 1.f;
        const uint32_t f2 = pack_bf16(fq, fq);
        float2 qz2 = make_float2(0.f, 0.f);   // phi(q').z, even and odd columns
        uint4 w[QCH];
#pragma unroll
        for (int j = 0; j < QCH; ++j)
          w[j] = *reinterpret_cast<const uint4 *>(st + kOffQ + chunk_off(tq, cb * QCH + j));
        uint32_t pk[4 * QCH];
#pragma unroll
        for (int j = 0; j < QCH; ++j) {
          uint32_t e[4] = {w[j].x, w[j].y, w[j].z, w[j].w};
          const float4 za = *reinterpret_cast<const float4 *>(zs + (cb * QCH + j) * 8);
          const float4 zb = *reinterpret_cast<const float4 *>(zs + (cb * QCH + j) * 8 + 4);
          const float zz[8] = {za.x, za.y, za.z, za.w, zb.x, zb.y, zb.z, zb.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            if (!ident) e[i] = phi_bf16x2(e[i]);
            e[i] = mul_bf16x2(e[i], f2);
            qz2 = ffma2(make_float2(bf_lo(e[i]), bf_hi(e[i])), make_float2(zz[2 * i], zz[2 * i + 1]),
                        qz2);
            pk[4 * j + i] = e[i];
          }
        }
        if constexpr (QCH == 4) tmem_st_32x32b_x16(tq_col(s), pk);
        else tmem_st_32x32b_x8(tq_col(s), pk);
        // factored: phi(q') . z~; explicit: lambda^(t+1) phi(q) . z.  The
        // part of this column block goes into the q bytes this thread alone
        // has read (the score epilogue sums the four parts of the row).
        *reinterpret_cast<float *>(st + kOffQ + chunk_off(tq, cb * QCH)) =
            (qz2.x + qz2.y) * (factored ? 1.f : (tq < Cv ? pw[tq + 1] : 0.f));
      }
      // (2) k: feature map, decay weights (factored), column sums for z
      // factored k weight lambda^(n_f - 1 - p) = Fk lambda^(C - 1 - s)
      // the k tile has its own ring: every warp checks that it has landed
      {
        bool okk = true;
        if (lane == 0) okk = mbar_wait(bar(kFullK0 + s), (c >> 1) & 1);
        if (!__shfl_sync(0xffffffffu, okk, 0)) {
          rf = 1;
          fail();
        }
      }
      if (kwarp) {
        float csum[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) csum[e] = 0.f;
        // every load of the thread's rows in flight before the first store
        uint4 w[RPL];
#pragma unroll
        for (int i = 0; i < RPL; ++i)
          w[i] = *reinterpret_cast<const uint4 *>(st + kOffK + chunk_off(lane + 32 * i, cg));
#pragma unroll
        for (int i = 0; i < RPL; ++i) {
          const int row = lane + 32 * i;
          const float wk = row < Cv ? pw[Cv - 1 - row] : 0.f;
          const float fk = row < Cv ? (factored ? Fk * pw[C - 1 - row] : 1.f) : 0.f;
          const uint32_t f2 = pack_bf16(fk, fk);
          uint32_t e[4] = {w[i].x, w[i].y, w[i].z, w[i].w};
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            if (!ident) e[q4] = phi_bf16x2(e[q4]);
            e[q4] = mul_bf16x2(e[q4], f2);
            // the explicit path keeps phi(k) unweighted for the score MMA; the
            // normaliser takes the weights here
            const float m = factored ? 1.f : wk;
            const float2 c2 = ffma2(make_float2(bf_lo(e[q4]), bf_hi(e[q4])), make_float2(m, m),
                                    make_float2(csum[2 * q4], csum[2 * q4 + 1]));
            csum[2 * q4] = c2.x;
            csum[2 * q4 + 1] = c2.y;
          }
          w[i] = make_uint4(e[0], e[1], e[2], e[3]);
        }
#pragma unroll
        for (int i = 0; i < RPL; ++i)
          *reinterpret_cast<uint4 *>(st + kOffK + chunk_off(lane + 32 * i, cg)) = w[i];
        ztot = warp_sum8_transposed(csum, lane);
      }
      fence_proxy_async_smem();
      tmem_wait_st();
      tc_fence_before();
      named_bar_sync(kBarPhi, kPhiThreads);
      if (tt == kPollPhi) {
        mbar_arrive(bar(kPhi0 + s));
        mbar_arrive(bar(kDenQz0 + c % kDenBufs));
      }
      if (!factored) {
        // after the score MMA: q rows (TMEM) times lambda^(t+1), k rows (SMEM)
        // times lambda^(Cv-1-s)
        if (tt == kPollPhi) check(mbar_wait(bar(kScore), c & 1));
        named_bar_sync(kBarPhi, kPhiThreads);
        if (rf) break;
        tc_fence_after();
        {
          const float f = tq < Cv ? pw[tq + 1] : 0.f;
          const uint32_t f2 = pack_bf16(f, f);
          uint32_t pk[4 * QCH];
          if constexpr (QCH == 4) tmem_ld_32x32b_x16(tq_col(s), pk);
          else tmem_ld_32x32b_x8(tq_col(s), pk);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 4 * QCH; ++i) pk[i] = mul_bf16x2(pk[i], f2);
          if constexpr (QCH == 4) tmem_st_32x32b_x16(tq_col(s), pk);
          else tmem_st_32x32b_x8(tq_col(s), pk);
        }
        {
          const float f = tq < Cv ? pw[Cv - 1 - tq] : 0.f;
          const uint32_t f2 = pack_bf16(f, f);
#pragma unroll
          for (int j = 0; j < QCH; ++j) {
            uint4 *p = reinterpret_cast<uint4 *>(st + kOffK + chunk_off(tq, cb * QCH + j));
            uint4 w = *p;
            *p = make_uint4(mul_bf16x2(w.x, f2), mul_bf16x2(w.y, f2), mul_bf16x2(w.z, f2),
                            mul_bf16x2(w.w, f2));
          }
        }
        tmem_wait_st();
        tc_fence_before();
        fence_proxy_async_smem();
        named_bar_sync(kBarPhi, kPhiThreads);
        if (tt == kPollPhi) mbar_arrive(bar(kRescale));
      }
    }
    // the last chunk's column sums; factored: z = lambda^(tokens since the frame start) z~
    if (!rf && nchunks > 0 && zowner)
      zs[zcol] = factored ? (zs[zcol] + ztot) * (Eq * pw[Cv_of(nchunks - 1)])
                          : pw[Cv_of(nchunks - 1)] * zs[zcol] + ztot;
    named_bar_sync(kBarPhi, kPhiThreads);
    if (!rf && last_seg && z_final && tt < DK) z_final[pair * DK + tt] = zs[tt];
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmCols);
  }
}

// ---------------------------------------------------------------------------
// State pass: for segment g of each head (tokens [g len, min(N, (g+1) len))),
// the segment's own final state from zero,
//   dS_g = sum_s lambda^(n-1-s) phi(k_s) v_s^T,  dz_g = sum_s lambda^(n-1-s) phi(k_s)
// (s and n counted inside the segment), written to slot pair * slots + g of
// out_S / out_z.  The segmented forward runs it on its first G - 1 segments
// (slots = G; the combine scan then turns the slots into starting states);
// linattn_causal_state runs it on whole sequences (one segment, slots = 1).
// Every k row is weighted by its own lambda^(n-1-s) (at most 1; weights below
// the fp32 range flush to zero, far below the rounding of the kept terms), so
// the state MMAs accumulate the whole segment with no decay step between
// chunks.
// Roles (768 threads): warp 0 TMA (k and v, 3 stages), warp 1 MMA issuer,
// warps 4-7 store of the final state, warps 8-23 feature map.
namespace sp {
constexpr int NT = 768;
constexpr int kStages = 3;
constexpr uint32_t kOffK = 0, kOffV = 2 * kPanel;
constexpr uint32_t kStage = 4 * kPanel;                  // 64 KB
constexpr uint32_t kOffMisc = kStages * kStage;          // 192 KB
constexpr uint32_t kMiscTmem = 256, kMiscAbort = 260, kMiscRoleFail = 272;
constexpr uint32_t kMiscPw = 320, kMiscZ = 848;
constexpr uint32_t kSmemBytes = kOffMisc + kMiscZ + 128 * 4;
static_assert(kSmemBytes <= 232448, "exceeds the per-CTA shared memory of sm_100");
enum Bar { kFull0 = 0, kFree0 = 3, kPhi0 = 6, kState = 9, kNumBars };
constexpr int kBarPhi = 1, kBarStore = 2;
constexpr int kPhiThreads = 512;
}  // namespace sp

template <int DKP, int DVP>
__global__ void __launch_bounds__(sp::NT, 1)
    causal_seg_state_tc_kernel(const __grid_constant__ CUtensorMap tm_k,
                               const __grid_constant__ CUtensorMap tm_v,
                               const float *__restrict__ lam, float *__restrict__ out_S,
                               float *__restrict__ out_z, int H, int N, int seg_len, int nseg,
                               int slots, bool ident) {
  constexpr int DK = 64 * DKP, DV = 64 * DVP;
  constexpr int KCH = 8 * DKP;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *sm = smem_raw;
  const uint32_t sb = smem_u32(sm);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (sb & 1023u) {
    if (tid == 0) atomicOr(&g_status, kStatusWaitTimeout);
    return;
  }
  // the forward launched after this grid as its dependent may start its
  // first segments' CTAs now (they do not read this grid's output)
  grid_launch_dependents();
  const long pair = blockIdx.x / nseg;
  const int g = blockIdx.x % nseg;
  const long slot = pair * slots + g;
  const float L = lam ? lam[pair % H] : 1.f;
  const int n0 = g * seg_len;
  const int n1 = min(N, n0 + seg_len);
  const int nchunks = (n1 - n0 + C - 1) / C;
  const int Ct = (n1 - n0) - (nchunks - 1) * C;   // valid tokens of the last chunk
  auto Cv_of = [&](int c) { return c == nchunks - 1 ? Ct : C; };
  uint8_t *misc = sm + sp::kOffMisc;
  auto bar = [&](int i) { return sb + sp::kOffMisc + 8u * static_cast<uint32_t>(i); };
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(misc + sp::kMiscTmem);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(misc + sp::kMiscAbort);
  volatile int *role_fail = reinterpret_cast<volatile int *>(misc + sp::kMiscRoleFail);
  float *pw = reinterpret_cast<float *>(misc + sp::kMiscPw);
  float *zs = reinterpret_cast<float *>(misc + sp::kMiscZ);
  if (tid == 0) {
    for (int i = 0; i < sp::kNumBars; ++i) mbar_init(bar(i), 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (tid < 4) role_fail[tid] = 0;
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 128);
    tmem_relinquish();
  }
  if (tid <= C) pw[tid] = pow_int(L, tid);
  if (tid < 128) zs[tid] = 0.f;
  if (DKP == 1)
    for (uint32_t o = tid * 16u; o < sp::kStages * kPanel; o += sp::NT * 16u)
      *reinterpret_cast<uint4 *>(sm + (o / kPanel) * sp::kStage + sp::kOffK + kPanel + o % kPanel) =
          make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  auto fail = [&]() { *abort_flag = 1; };

  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;
      for (int c = 0; c < nchunks && !*abort_flag; ++c) {
        const int s = c % sp::kStages;
        if (c >= sp::kStages &&
            !mbar_wait_backoff(bar(sp::kFree0 + s), ((c - sp::kStages) / sp::kStages) & 1)) {
          fail();
          break;
        }
        const uint32_t base = sb + s * sp::kStage;
        const uint32_t b = bar(sp::kFull0 + s);
        const int y = n0 + c * C;
        mbar_arrive_expect_tx(b, (DKP + DVP) * kPanel);
        for (int p = 0; p < DKP; ++p)
          tma_load_3d(base + sp::kOffK + p * kPanel, &tm_k, b, 64 * p, y, static_cast<int>(pair));
        for (int p = 0; p < DVP; ++p)
          tma_load_3d(base + sp::kOffV + p * kPanel, &tm_v, b, 64 * p, y, static_cast<int>(pair));
        if (c + sp::kStages < nchunks) {
          for (int p = 0; p < DKP; ++p)
            tma_prefetch_l2_3d(&tm_k, 64 * p, y + sp::kStages * C, static_cast<int>(pair));
          for (int p = 0; p < DVP; ++p)
            tma_prefetch_l2_3d(&tm_v, 64 * p, y + sp::kStages * C, static_cast<int>(pair));
        }
        issued = c + 1;
      }
      if (*abort_flag)
        for (int c = issued - sp::kStages < 0 ? 0 : issued - sp::kStages; c < issued; ++c)
          mbar_wait(bar(sp::kFull0 + c % sp::kStages), (c / sp::kStages) & 1);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16(128, DV, 1, 1);
      bool ok = true;
      for (int c = 0; ok && c < nchunks; ++c) {
        const int s = c % sp::kStages;
        const uint32_t st = sb + s * sp::kStage;
        if (*abort_flag || !mbar_wait(bar(sp::kPhi0 + s), (c / sp::kStages) & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t k0 = sdesc_sw128(st + sp::kOffK, kPanel, 1024);
        const uint64_t v0 = sdesc_sw128(st + sp::kOffV, kPanel, 1024);
#pragma unroll
        for (int ks = 0; ks < C / 16; ++ks)
          umma_bf16(tmem, k0 + ks * (2048 >> 4), v0 + ks * (2048 >> 4), idS,
                    (c > 0 || ks > 0) ? 1u : 0u);
        umma_commit(bar(sp::kFree0 + s));
      }
      if (!ok) fail();
      // every MMA done: the state is final (and TMEM idle before teardown)
      umma_commit(bar(sp::kState));
      mbar_wait(bar(sp::kState), 0);
    }
    __syncwarp();
  } else if (warp >= 4 && warp < 8) {
    const int wq = warp - 4;
    const int r = wq * 32 + lane;
    const uint32_t lf = static_cast<uint32_t>(wq * 32) << 16;
    // one thread polls for the whole pass, sleeping between tries (warp 7,
    // away from the TMA and feature-map pollers' schedulers); the others wait
    // at the named barrier
    if (r == 96 && (*abort_flag || !mbar_wait_backoff(bar(sp::kState), 0, 512))) fail();
    named_bar_sync(sp::kBarStore, 128);
    tc_fence_after();
    if (!*abort_flag) {
#pragma unroll 1
      for (int blk = 0; blk < DV / 32; ++blk) {
        uint32_t sv[32];
        tmem_ld_32x32b_x32(tmem + lf + blk * 32, sv);   // warp-wide load
        tmem_wait_ld();
        if (r < DK) {
          float4 *dst =
              reinterpret_cast<float4 *>(out_S + (slot * DK + r) * static_cast<long>(DV)) + blk * 8;
#pragma unroll
          for (int i = 0; i < 8; ++i)
            dst[i] = nchunks == 0 ? make_float4(0.f, 0.f, 0.f, 0.f)
                                  : make_float4(__uint_as_float(sv[4 * i]),
                                                __uint_as_float(sv[4 * i + 1]),
                                                __uint_as_float(sv[4 * i + 2]),
                                                __uint_as_float(sv[4 * i + 3]));
        }
      }
    }
    tc_fence_before();
  } else if (warp >= 8) {
    const int tt = tid - 256;                 // 0..511
    const int fw = tt >> 5;                   // feature-map warp 0..15
    volatile int &rf = role_fail[1];
    // a warp owns one column group of 8 columns over all 128 rows (the column
    // sums of z need no atomics); with d_k = 64 only the first 8 warps work
    constexpr int NCG = KCH, RPL = 128 / 32;
    const bool kwarp = fw < NCG;
    const int cg = fw;
    float ztot = 0.f;
    const int zcol = cg * 8 + warp_sum8_index(lane);
    const bool zowner = kwarp && (lane & 3) == 0;
    const float log2L = L > 0.f ? log2f(L) : 0.f;
    for (int c = 0; c < nchunks; ++c) {
      const int s = c % sp::kStages;
      uint8_t *st = sm + s * sp::kStage;
      // the previous chunk's column sums (already weighted to the segment end)
      if (c > 0 && zowner) zs[zcol] += ztot;
      if (tt == 32 && (*abort_flag || !mbar_wait(bar(sp::kFull0 + s), (c / sp::kStages) & 1))) {
        rf = 1;
        fail();
      }
      named_bar_sync(sp::kBarPhi, sp::kPhiThreads);
      if (rf) break;
      const int Cv = Cv_of(c);
      // lambda^(tokens of the segment after this chunk)
      const int after = (n1 - n0) - c * C - Cv;
      const float Tc = after == 0 ? 1.f : (L > 0.f ? exp2f(static_cast<float>(after) * log2L) : 0.f);
      if (kwarp) {
        float csum[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) csum[e] = 0.f;
        uint4 w[RPL];
#pragma unroll
        for (int i = 0; i < RPL; ++i)
          w[i] = *reinterpret_cast<const uint4 *>(st + sp::kOffK + chunk_off(lane + 32 * i, cg));
#pragma unroll
        for (int i = 0; i < RPL; ++i) {
          const int row = lane + 32 * i;
          const float wk = row < Cv ? Tc * pw[Cv - 1 - row] : 0.f;
          const uint32_t f2 = pack_bf16(wk, wk);
          uint32_t e[4] = {w[i].x, w[i].y, w[i].z, w[i].w};
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            if (!ident) e[q4] = phi_bf16x2(e[q4]);
            e[q4] = mul_bf16x2(e[q4], f2);
            csum[2 * q4] += bf_lo(e[q4]);
            csum[2 * q4 + 1] += bf_hi(e[q4]);
          }
          w[i] = make_uint4(e[0], e[1], e[2], e[3]);
        }
#pragma unroll
        for (int i = 0; i < RPL; ++i)
          *reinterpret_cast<uint4 *>(st + sp::kOffK + chunk_off(lane + 32 * i, cg)) = w[i];
        ztot = warp_sum8_transposed(csum, lane);
      }
      fence_proxy_async_smem();
      named_bar_sync(sp::kBarPhi, sp::kPhiThreads);
      if (tt == 32) mbar_arrive(bar(sp::kPhi0 + s));
    }
    if (!rf && nchunks > 0 && zowner) zs[zcol] += ztot;
    named_bar_sync(sp::kBarPhi, sp::kPhiThreads);
    if (!rf && tt < DK) out_z[slot * DK + tt] = zs[tt];
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

}  // namespace stc
}  // namespace linattn
