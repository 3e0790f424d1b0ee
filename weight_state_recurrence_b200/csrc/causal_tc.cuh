// Chunked causal forward on the 5th-generation tensor cores (bf16 operands,
// fp32 accumulators in TMEM), d_k = 128 or 64, dv sliced 64 columns per CTA.
// With d_k = 64 the operand tiles keep their 128-column shape: the second
// d_k panel of q and k is zero (loaded never, transformed never), so the score
// and O_x chains skip its K steps and the state rows 64-127 stay zero.
//
// The method (fast-weight article §2.1/§3.2/§4.2 recurrence, §3.1
// triangular-mask form, §4.1 note and §5.2 "cut the sequence into blocks:
// parallel inside a block, carried across blocks") written per chunk of
// C = 128 tokens, t and s 0-based inside the chunk, Cv valid tokens, state
// (S, z) carried from the previous chunk:
//
//   A      = (phi(Q) phi(K)^T) o M,       M[t][s] = lambda^(t-s) for s <= t, else 0
//   O_in   = A V,                         rs = A 1
//   O_x    = phi(Q) S,                    qz = phi(Q) z
//   y_t    = (O_in[t] + lambda^(t+1) O_x[t]) / (rs[t] + lambda^(t+1) qz[t] + eps)
//   S     <- lambda^Cv S + (Lk phi(K))^T V,   Lk = diag(lambda^(Cv-1-t))
//   z     <- lambda^Cv z + (Lk phi(K))^T 1
//
// Tensor-core work per chunk (M = 128, K = 16 per instruction; an
// instruction costs the same for every N up to 128, so the side products ride
// along as extra columns of the 64-wide ones):
//   A      N=128  phi(Q) x phi(K)^T                     K-major x K-major
//   O_x    N=80   phi(Q) x [S | 1, z_hi, z_lo]           K-major x MN-major
//   O_in   N=80   A(bf16) x [V | 1, ...]                 K-major x MN-major
//   S, z   N=80   (Lk phi(K))^T x [V | 1, ...]           MN-major x MN-major
// The "[.. | 1, z_hi, z_lo]" columns come from one shared 64-column operand
// atom (column 0 = ones, columns 1-2 = the normaliser as a bf16 hi/lo pair).
// They give the row sums of the bf16 score tile (so the denominator sums
// exactly the weights the numerator uses), phi(q).z with ~16 bits of z, and
// the update of z.  The fp32 state S and z live in TMEM for the whole
// sequence: after each chunk one warpgroup reads them, emits S as the bf16
// operand of the next O_x, and writes them back multiplied by lambda^Cv so the
// next state MMA accumulates onto the decayed state.
//
// Decay.  For lambda >= kFactorMin the decay is factored into the operands:
// phi(q_t) is scaled by lambda^(t+1-Cv) and phi(k_s) by lambda^(Cv-1-s) while
// the feature map is applied, so the score MMA yields lambda^(t-s)
// phi(q_t).phi(k_s) directly (the epilogue only masks s > t), the state MMA
// gets its weights for free, and the carried-state terms need the single
// factor lambda^Cv.  Smaller lambda (down to 0) uses the explicit form: the
// epilogue multiplies the score tile by lambda^(t-s) and the k tile is
// weighted by Lk in a second pass after the score MMA has read it.
//
// When dv = 128 the two CTAs that own the two 64-column halves of one head
// run as a 2-CTA cluster and share the feature-map work: each loads and
// transforms only its 64 rows of the chunk's q and k tiles and copies the
// transformed rows into its peer's shared memory with a bulk DSMEM copy
// (plain copies, no multicast), so phi is evaluated once per element.
//
// Warp roles (768 threads):
//   warp 0      TMA producer of the q/k tiles (this CTA's rows)
//   warp 1      TMEM owner and the single MMA-issuing thread
//   warp 2      TMA producer of the v tiles (each half of the 2-stage ring is
//               recycled on its own)
//   warps 3-7, 16-23  phi (and the factored decay scales) applied in place
//               to q and k tiles in packed bf16x2, one d_k half at a time so
//               the first half is copied to the peer and multiplied while
//               the second is transformed; explicit decay: the k weighting pass
//   warps 8-11  masked score tile: TMEM -> registers -> bf16 operand in SMEM
//   warps 12-15 state update, then the output y = numerator / denominator
// Every barrier wait is bounded (see sm100.cuh); a wait that runs out
// records an error flag and every role leaves its loop.
#pragma once
#include "common.cuh"
#include "sm100.cuh"

namespace linattn {
namespace tc {

constexpr int C = 128;      // tokens per chunk
constexpr int DK = 128;     // key dimension handled by this kernel
constexpr int DVS = 64;     // dv columns per CTA
constexpr int NT = 768;
constexpr int kPrefetch = 2;   // chunks ahead that the producers prefetch into L2

// phi transform: warps 3-7 and 16-23
constexpr int kXformThreads = 416;
constexpr int kBarXform = 1, kBarEpiA = 2, kBarOut = 3;  // named barrier ids

// ---- shared memory (offsets from the 1024-byte aligned dynamic base)
constexpr uint32_t kPanel = C * 128;            // 128 rows x 128 bytes
constexpr uint32_t kOffQ = 0;                   // per stage: phi(Q), 2 panels (d_k 0-63, 64-127)
constexpr uint32_t kOffK = 2 * kPanel;          //            phi(K), 2 panels
constexpr uint32_t kOffV = 4 * kPanel;          //            V slice, 1 panel
constexpr uint32_t kStage = 5 * kPanel;         // 80 KB
constexpr uint32_t kOffA = 2 * kStage;          // bf16 score tile, 2 panels (keys 0-63, 64-127)
constexpr uint32_t kOffS = kOffA + 2 * kPanel;  // bf16 S slice operand atom (MN-major)
constexpr uint32_t kOffX = kOffS + kPanel;      // shared atom: col 0 = 1, cols 1-2 = z hi/lo
constexpr uint32_t kOffMisc = kOffX + kPanel;
constexpr uint32_t kMiscBytes = 2944;
constexpr uint32_t kSmemBytes = kOffMisc + kMiscBytes;   // 232,320 bytes
static_assert(kSmemBytes <= 232448, "exceeds the per-CTA shared memory of sm_100");
constexpr uint32_t kQKTxBytes = 4 * kPanel;
constexpr uint32_t kVTxBytes = kPanel;

// ---- barriers (8 bytes each, at kOffMisc)
enum Bar {
  kFullQK0 = 0, kFullQK1, kFullV0, kFullV1, kFreeQK0, kFreeQK1, kFreeV0, kFreeV1,
  kPhi0, kPhi1, kPhiB0, kPhiB1, kAFull0, kAFull1, kAFree0, kAFree1,
  kAbfFull, kOvDone, kOxDone, kKsDone, kDsDone, kStateDone, kOutDone, kFinal,
  kPeerFree0, kPeerFree1,   // the peer CTA's q/k stage may be overwritten
  kNumBars
};
static_assert(kNumBars * 8 <= 256, "barrier area overflow");
constexpr uint32_t kMiscTmem = 256, kMiscAbort = 260, kMiscConsumed = 264;
// per-role failure flags (transform, score tile, output/state), see below
constexpr uint32_t kMiscRoleFail = 272;
constexpr uint32_t kMiscPw = 320;                    // lambda^i, i = 0..C      (132 floats)
constexpr uint32_t kMiscKf = kMiscPw + 132 * 4;      // lambda^(C-1-t)
constexpr uint32_t kMiscKt = kMiscKf + 128 * 4;      // lambda^(Ct-1-t), 0 past Ct
constexpr uint32_t kMiscQf = kMiscKt + 128 * 4;      // lambda^(t+1-C)   (factored decay)
constexpr uint32_t kMiscQt = kMiscQf + 128 * 4;      // lambda^(t+1-Ct), 0 past Ct
static_assert(kMiscQt + 128 * 4 <= kMiscBytes, "misc region overflow");

// Heads with lambda >= kFactorMin use the factored decay: the row scales
// lambda^(t+1-Cv) on phi(q) and lambda^(Cv-1-t) on phi(k) make the score MMA
// produce lambda^(t-s) phi(q_t).phi(k_s) directly and give the state update
// its weights; the largest scale, lambda^-(C-1), stays below 1e20.  Smaller
// lambda (down to 0) applies lambda^(t-s) to the score tile explicitly.
constexpr float kFactorMin = 0.7f;

// ---- tensor memory columns (fp32, lane = row)
constexpr uint32_t kTmA = 0;      // two 128-column score buffers
constexpr uint32_t kTmOX = 256;   // O_x (64) | phi(q).1 | qz_hi | qz_lo | ...   (80)
constexpr uint32_t kTmOV = 336;   // O_in (64) | row sum | ...                     (80)
constexpr uint32_t kTmS = 416;    // S (64) | z | zeros ...   lane = d_k row       (80)
constexpr uint32_t kTmCols = 512;

constexpr uint32_t kIdA = idesc_bf16(128, 128, 0, 0);
constexpr uint32_t kIdN80 = idesc_bf16(128, 80, 0, 1);    // K-major A, MN-major B
constexpr uint32_t kIdS = idesc_bf16(128, 80, 1, 1);      // MN-major A, MN-major B

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&p);
}

// phi on a packed pair: max(x,0) + 2^(min(x,0) log2 e), in bf16x2 arithmetic.
// log2 e is split into a bf16 head and tail so its rounding does not bias the
// exponent; ex2 takes the bf16 argument (the result is bf16 either way).
__device__ __forceinline__ uint32_t phi_bf16x2(uint32_t x) {
  const uint32_t zero = 0u;
  const uint32_t l2e_hi = 0x3FB93FB9u;   // bf16(log2 e) = 1.4453125, twice
  const uint32_t l2e_lo = 0xBB2CBB2Cu;   // bf16(log2 e - 1.4453125) = -0.00262451, twice
  uint32_t m, r, t, e, y;
  asm("min.bf16x2 %0, %1, %2;" : "=r"(m) : "r"(x), "r"(zero));
  asm("max.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(x), "r"(zero));
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(t) : "r"(m), "r"(l2e_hi));
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(t) : "r"(m), "r"(l2e_lo), "r"(t));
  asm("ex2.approx.ftz.bf16x2 %0, %1;" : "=r"(e) : "r"(t));
  asm("add.rn.bf16x2 %0, %1, %2;" : "=r"(y) : "r"(r), "r"(e));
  return y;
}

__device__ __forceinline__ uint32_t mul_bf16x2(uint32_t x, uint32_t s2) {
  uint32_t y;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(y) : "r"(x), "r"(s2));
  return y;
}

// K-major operand tile [n rows x 128] with 128B swizzle, 2 panels of 64
// columns, panel stride `panel_bytes`: byte offset of element (row, col).
__device__ __forceinline__ uint32_t kmajor_off(uint32_t row, uint32_t col, uint32_t panel_bytes) {
  return (col >> 6) * panel_bytes + sw128_offset(row, (col & 63) * 2);
}

// Elementwise pass over `bytes` of a shared tile by `nthr` threads, U
// independent 16-byte chunks in flight per thread.  The tile is a list of
// equal blocks: block b starts at p + b * block_stride and is block_bytes
// long.  op(word, byte_offset_from_p) returns the new 32-bit word (two bf16).
template <int U, typename Op>
__device__ __forceinline__ void tile_pass(uint8_t *p, uint32_t block_bytes, uint32_t block_stride,
                                          int nblocks, int tid, int nthr, Op op) {
  const uint32_t step = static_cast<uint32_t>(nthr) * 16u;
  const uint32_t total = block_bytes * static_cast<uint32_t>(nblocks);
  auto addr = [&](uint32_t lin) { return (lin / block_bytes) * block_stride + lin % block_bytes; };
  for (uint32_t o0 = static_cast<uint32_t>(tid) * 16u; o0 < total; o0 += U * step) {
    uint4 w[U];
#pragma unroll
    for (int i = 0; i < U; ++i)
      if (o0 + i * step < total) w[i] = *reinterpret_cast<const uint4 *>(p + addr(o0 + i * step));
#pragma unroll
    for (int i = 0; i < U; ++i) {
      const uint32_t o = addr(o0 + i * step);
      w[i].x = op(w[i].x, o);
      w[i].y = op(w[i].y, o);
      w[i].z = op(w[i].z, o);
      w[i].w = op(w[i].w, o);
    }
#pragma unroll
    for (int i = 0; i < U; ++i)
      if (o0 + i * step < total) *reinterpret_cast<uint4 *>(p + addr(o0 + i * step)) = w[i];
  }
}

// phi over this CTA's rows of `nblocks` panels `stride` bytes apart (a q
// panel and the k panel 2 panels further on), in place, U 16-byte chunks in
// flight per thread.  With `scaled`, rows of q panels (offset < 2 panels) are
// multiplied by qsc[t] and rows of k panels by ksc[t] (the factored decay); a
// 16-byte chunk never straddles two rows.
template <int U>
__device__ __forceinline__ void phi_pass(uint8_t *p, uint32_t own_bytes, uint32_t stride,
                                         int nblocks, int row0, const float *qsc,
                                         const float *ksc, bool scaled, bool ident, int tid,
                                         int nthr) {
  const uint32_t step = static_cast<uint32_t>(nthr) * 16u;
  const uint32_t total = own_bytes * static_cast<uint32_t>(nblocks);
  for (uint32_t o0 = static_cast<uint32_t>(tid) * 16u; o0 < total; o0 += U * step) {
    uint4 w[U];
    uint32_t off[U];
#pragma unroll
    for (int i = 0; i < U; ++i) {
      const uint32_t lin = o0 + i * step;
      off[i] = (lin / own_bytes) * stride + lin % own_bytes;
      if (lin < total) w[i] = *reinterpret_cast<const uint4 *>(p + off[i]);
    }
#pragma unroll
    for (int i = 0; i < U; ++i) {
      if (!ident) {
        w[i].x = phi_bf16x2(w[i].x);
        w[i].y = phi_bf16x2(w[i].y);
        w[i].z = phi_bf16x2(w[i].z);
        w[i].w = phi_bf16x2(w[i].w);
      }
      if (scaled) {
        const uint32_t row = static_cast<uint32_t>(row0) + ((off[i] % kPanel) >> 7);
        const float f = (off[i] < 2 * kPanel ? qsc : ksc)[row];
        const uint32_t f2 = pack_bf16(f, f);
        w[i].x = mul_bf16x2(w[i].x, f2);
        w[i].y = mul_bf16x2(w[i].y, f2);
        w[i].z = mul_bf16x2(w[i].z, f2);
        w[i].w = mul_bf16x2(w[i].w, f2);
      }
    }
#pragma unroll
    for (int i = 0; i < U; ++i)
      if (o0 + i * step < total) *reinterpret_cast<uint4 *>(p + off[i]) = w[i];
  }
}

template <bool kPair, bool kDk64>
__global__ void __launch_bounds__(NT, 1)
    causal_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                     const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const float *__restrict__ lam,
                     float eps, const float *__restrict__ S_init, const float *__restrict__ z_init,
                     __nv_bfloat16 *__restrict__ out, float *__restrict__ S_final,
                     float *__restrict__ z_final, int H, int N, int DV, bool ident) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *sm = smem_raw;
  const uint32_t sb = smem_u32(sm);
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  // The swizzled operand tiles need a 1024-byte aligned base (this kernel has
  // no static shared memory, so the dynamic base is aligned); refuse otherwise.
  if (sb & 1023u) {
    if (tid == 0) atomicOr(&g_status, kStatusWaitTimeout);
    return;
  }
  const int nslices = DV / DVS;
  const int pair = blockIdx.x / nslices;
  const int j0 = (blockIdx.x % nslices) * DVS;
  // with a peer, this CTA owns rows [row0, row0 + 64) of every q/k tile
  const uint32_t rank = kPair ? cluster_ctarank() : 0u;
  const uint32_t peer = rank ^ 1u;
  const int row0 = kPair ? static_cast<int>(rank) * 64 : 0;
  const uint32_t own_off = static_cast<uint32_t>(row0) * 128u;   // byte offset inside a panel
  const uint32_t own_bytes = kPair ? kPanel / 2 : kPanel;        // own rows of one panel
  const int h = pair % H;
  const float L = lam ? lam[h] : 1.f;
  const int nchunks = (N + C - 1) / C;
  const int Ct = N - (nchunks - 1) * C;  // valid tokens of the last chunk

  uint8_t *misc = sm + kOffMisc;
  auto bar = [&](int i) { return sb + kOffMisc + 8u * static_cast<uint32_t>(i); };
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(misc + kMiscTmem);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(misc + kMiscAbort);
  volatile int *consumed = reinterpret_cast<volatile int *>(misc + kMiscConsumed);
  float *pw = reinterpret_cast<float *>(misc + kMiscPw);
  float *kf = reinterpret_cast<float *>(misc + kMiscKf);
  float *kt = reinterpret_cast<float *>(misc + kMiscKt);
  float *qf = reinterpret_cast<float *>(misc + kMiscQf);
  float *qt = reinterpret_cast<float *>(misc + kMiscQt);
  const bool factored = L >= kFactorMin;   // uniform over the CTA (and its peer)
  constexpr bool dk64 = kDk64;             // only the first d_k panel holds data
  constexpr int kpanels = kDk64 ? 1 : 2;
  constexpr int dk = kDk64 ? 64 : DK;      // the caller's d_k (state layout)

  // ------------------------------------------------------------ set-up
  if (tid == 0) {
    for (int i = 0; i < kNumBars; ++i) mbar_init(bar(i), 1);
    *abort_flag = 0;
    *consumed = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmCols);
    tmem_relinquish();
  }
  if (tid <= C) pw[tid] = pow_int(L, tid);
  // operand tiles that start as constants: S = 0; the shared atom with
  // column 0 = ones and z = 0; the score tile's blocks above the diagonal
  // (always zero)
  for (uint32_t o = tid * 16u; o < kPanel; o += NT * 16u) {
    *reinterpret_cast<uint4 *>(sm + kOffS + o) = make_uint4(0, 0, 0, 0);
    *reinterpret_cast<uint4 *>(sm + kOffX + o) = make_uint4(0, 0, 0, 0);
  }
  for (uint32_t o = tid * 16u; o < 2 * kPanel; o += NT * 16u)
    *reinterpret_cast<uint4 *>(sm + kOffA + o) = make_uint4(0, 0, 0, 0);
  if (dk64)   // the second d_k panel of the q and k tiles of both stages stays zero
    for (uint32_t o = tid * 16u; o < 4 * kPanel; o += NT * 16u) {
      const uint32_t st = (o / (2 * kPanel)) * kStage, w = o % (2 * kPanel);
      *reinterpret_cast<uint4 *>(sm + st + (w < kPanel ? kOffQ : kOffK - kPanel) + kPanel + w) =
          make_uint4(0, 0, 0, 0);
    }
  __syncthreads();
  if (tid < C) {
    *reinterpret_cast<__nv_bfloat16 *>(sm + kOffX + sw128_offset(tid, 0)) =
        __float2bfloat16_rn(1.f);
    kf[tid] = pw[C - 1 - tid];
    kt[tid] = tid < Ct ? pw[Ct - 1 - tid] : 0.f;
    qf[tid] = factored ? 1.f / pw[C - 1 - tid] : 0.f;
    qt[tid] = factored && tid < Ct ? 1.f / pw[Ct - 1 - tid] : 0.f;
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  if (kPair) cluster_sync_all();   // the peer's barriers are initialised before any remote use
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // A caller-supplied starting state: the state warpgroup puts lambda^Cv S_init
  // (and z) into the TMEM state, where the first state MMA accumulates onto
  // it, and S_init, z_init into the operands of the first O_x MMA.
  const bool has_init = S_init != nullptr;
  if (has_init) {
    if (warp >= 12 && warp < 16) {
      const int r = (warp - 12) * 32 + lane;   // d_k row
      const bool live = !kDk64 || r < dk;
      const uint32_t lane_field = static_cast<uint32_t>((warp - 12) * 32) << 16;
      const float g0 = pw[nchunks == 1 ? Ct : C];   // decay of the first chunk
      const float4 *src = reinterpret_cast<const float4 *>(
          S_init + (static_cast<long>(pair) * dk + (live ? r : 0)) * DV + j0);
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t sv[32], pk[16];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float4 f = live ? src[half * 8 + i] : make_float4(0.f, 0.f, 0.f, 0.f);
          sv[4 * i] = __float_as_uint(f.x * g0);
          sv[4 * i + 1] = __float_as_uint(f.y * g0);
          sv[4 * i + 2] = __float_as_uint(f.z * g0);
          sv[4 * i + 3] = __float_as_uint(f.w * g0);
          pk[2 * i] = pack_bf16(f.x, f.y);
          pk[2 * i + 1] = pack_bf16(f.z, f.w);
        }
        tmem_st_32x32b_x32(tmem + lane_field + kTmS + half * 32, sv);
#pragma unroll
        for (int i = 0; i < 4; ++i)
          *reinterpret_cast<uint4 *>(sm + kOffS + sw128_offset(r, half * 64 + i * 16)) =
              make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
      }
      const float z0 = live ? z_init[static_cast<long>(pair) * dk + r] : 0.f;
      uint32_t zcol[16];
      zcol[0] = __float_as_uint(z0 * g0);
#pragma unroll
      for (int i = 1; i < 16; ++i) zcol[i] = 0u;
      tmem_st_32x32b_x16(tmem + lane_field + kTmS + 64, zcol);
      tmem_wait_st();
      const __nv_bfloat16 zh = __float2bfloat16_rn(z0);
      const __nv_bfloat16 zl = __float2bfloat16_rn(z0 - __bfloat162float(zh));
      *reinterpret_cast<__nv_bfloat16 *>(sm + kOffX + sw128_offset(r, 2)) = zh;
      *reinterpret_cast<__nv_bfloat16 *>(sm + kOffX + sw128_offset(r, 4)) = zl;
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }

  auto fail = [&]() { *abort_flag = 1; };
  // Roles with several warps meet at a named barrier once per step.  A
  // failed wait sets the role's shared flag (and the kernel-wide one) before
  // that barrier; every thread reads the role flag after it, so the whole role
  // leaves its loop together and no thread is left waiting at a barrier.
  volatile int *role_fail = reinterpret_cast<volatile int *>(misc + kMiscRoleFail);
  if (tid < 4) role_fail[tid] = 0;
  __syncthreads();

  if (warp == 0 || warp == 2) {
    // ------------------------------------------------------ TMA producers
    if (lane == 0) {
      const bool qk = warp == 0;
      int issued = 0;
      for (int c = 0; c < nchunks && !*abort_flag; ++c) {
        const int s = c & 1;
        if (c >= 2 && !mbar_wait(bar((qk ? kFreeQK0 : kFreeV0) + s), ((c - 2) >> 1) & 1)) {
          fail();
          break;
        }
        const uint32_t base = sb + s * kStage;
        if (qk) {
          // this CTA's MMAs are done with the stage: the peer may write its rows into it
          if (kPair && c >= 2) mbar_arrive_remote(map_to_rank(bar(kPeerFree0 + s), peer));
          const uint32_t b = bar(kFullQK0 + s);
          mbar_arrive_expect_tx(b, (kPair ? kQKTxBytes / 2 : kQKTxBytes) / (dk64 ? 2 : 1));
          const int y = c * C + row0;
          tma_load_3d(base + kOffQ + own_off, &tm_q, b, 0, y, pair);
          tma_load_3d(base + kOffK + own_off, &tm_k, b, 0, y, pair);
          if (!dk64) {
            tma_load_3d(base + kOffQ + kPanel + own_off, &tm_q, b, 64, y, pair);
            tma_load_3d(base + kOffK + kPanel + own_off, &tm_k, b, 64, y, pair);
          }
          // the same rows two chunks ahead into L2, so that their load, issued
          // when this stage frees up again, does not wait on HBM
          if (c + kPrefetch < nchunks) {
            const int yp = y + kPrefetch * C;
            tma_prefetch_l2_3d(&tm_q, 0, yp, pair);
            tma_prefetch_l2_3d(&tm_k, 0, yp, pair);
            if (!dk64) {
              tma_prefetch_l2_3d(&tm_q, 64, yp, pair);
              tma_prefetch_l2_3d(&tm_k, 64, yp, pair);
            }
          }
        } else {
          const uint32_t b = bar(kFullV0 + s);
          mbar_arrive_expect_tx(b, kVTxBytes);
          tma_load_3d(base + kOffV, &tm_v, b, j0, c * C, pair);
          if (c + kPrefetch < nchunks) tma_prefetch_l2_3d(&tm_v, j0, (c + kPrefetch) * C, pair);
        }
        issued = c + 1;
      }
      if (*abort_flag) {
        // let every copy this thread started land before the CTA exits
        if (qk) {
          for (int c = *consumed; c < issued; ++c)
            mbar_wait(bar(kFullQK0 + (c & 1)), (c >> 1) & 1);
        } else {
          for (int c = issued - 2 < 0 ? 0 : issued - 2; c < issued; ++c)
            mbar_wait(bar(kFullV0 + (c & 1)), (c >> 1) & 1);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      auto mma_scores = [&](int c) -> bool {
        const int s = c & 1;
        if (c >= 2 && !mbar_wait(bar(kAFree0 + s), ((c - 2) >> 1) & 1)) return false;
        const uint32_t st = sb + s * kStage;
#pragma unroll
        for (int ks = 0; ks < DK / 16; ++ks) {
          if (ks >= 4 * kpanels) break;   // the zero second panel adds nothing
          // d_k half 0 (ks < 4) and half 1 become ready separately
          if ((ks & 3) == 0) {
            if (!mbar_wait(bar((ks == 0 ? kPhi0 : kPhiB0) + s), (c >> 1) & 1)) return false;
            tc_fence_after();
          }
          const uint32_t off = (ks >> 2) * kPanel + (ks & 3) * 32;
          umma_bf16(tmem + kTmA + s * 128, sdesc_sw128(st + kOffQ + off, 16, 1024),
                    sdesc_sw128(st + kOffK + off, 16, 1024), kIdA, ks > 0);
        }
        umma_commit(bar(kAFull0 + s));
        return true;
      };
      bool ok = nchunks > 0 && mma_scores(0);
      for (int c = 0; ok && c < nchunks; ++c) {
        const int s = c & 1;
        const uint32_t st = sb + s * kStage;
        if (*abort_flag) break;
        const uint32_t va = st + kOffV;
        const uint32_t xa = sb + kOffX;
        // [S | z] += (Lk phi(K))^T [V | 1]   (onto the state decayed by lambda^Cv)
        if ((!factored && !mbar_wait(bar(kKsDone), c & 1)) ||
            !mbar_wait(bar(kFullV0 + s), (c >> 1) & 1) ||
            (c >= 1 && !mbar_wait(bar(kStateDone), (c - 1) & 1))) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < C / 16; ++ks)
          umma_bf16(tmem + kTmS, sdesc_sw128(st + kOffK + ks * 2048, kPanel, 1024),
                    sdesc_sw128(va + ks * 2048, xa - va, 1024), kIdS,
                    (c > 0 || ks > 0 || has_init) ? 1u : 0u);
        umma_commit(bar(kDsDone));
        // [O_x | . | qz] = phi(Q) [S | 1, z_hi, z_lo]   (state before this chunk)
        if (c >= 1 && !mbar_wait(bar(kOutDone), (c - 1) & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < DK / 16; ++ks) {
          if (ks >= 4 * kpanels) break;
          const uint32_t off = (ks >> 2) * kPanel + (ks & 3) * 32;
          umma_bf16(tmem + kTmOX, sdesc_sw128(st + kOffQ + off, 16, 1024),
                    sdesc_sw128(sb + kOffS + ks * 2048, kOffX - kOffS, 1024), kIdN80, ks > 0);
        }
        umma_commit(bar(kOxDone));
        umma_commit(bar(kFreeQK0 + s));   // q/k tiles of this chunk fully consumed
        // [O_in | rs] = A [V | 1]
        if (!mbar_wait(bar(kAbfFull), c & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < C / 16; ++ks)
          umma_bf16(tmem + kTmOV,
                    sdesc_sw128(sb + kOffA + (ks >> 2) * kPanel + (ks & 3) * 32, 16, 1024),
                    sdesc_sw128(va + ks * 2048, xa - va, 1024), kIdN80, ks > 0);
        umma_commit(bar(kOvDone));
        umma_commit(bar(kFreeV0 + s));    // v tile of this chunk fully consumed
        if (c + 1 < nchunks && !(ok = mma_scores(c + 1))) break;
      }
      if (!ok) fail();
      // make sure nothing this thread issued is still running
      umma_commit(bar(kFinal));
      mbar_wait(bar(kFinal), 0);
    }
    __syncwarp();
  } else if (warp < 8 || warp >= 16) {
    // ------------------------------------- phi transform, phi(k) weighting
    const int tt = warp < 8 ? tid - 96 : tid - 512 + 160;
    volatile int &rf = role_fail[0];
    auto check = [&](bool ok_wait) {
      if (!ok_wait || *abort_flag) {
        rf = 1;
        fail();
      }
    };
    // returns false when the role must stop (same answer in every thread)
    auto transform = [&](int c) -> bool {
      const int s = c & 1;
      check(mbar_wait(bar(kFullQK0 + s), (c >> 1) & 1));
      if (tt == 0) *consumed = c + 1;
      // the peer's MMAs must be done with its copy of this stage before we copy into it
      if (kPair && tt == 0 && c >= 2) check(mbar_wait(bar(kPeerFree0 + s), ((c - 2) >> 1) & 1));
      // this CTA's rows, one d_k half (q panel g and k panel g) at a time
      const bool tail = c == nchunks - 1;
      for (int g = 0; g < kpanels; ++g) {
        uint8_t *base = sm + s * kStage + kOffQ + g * kPanel;
        if (!rf && (factored || !ident))
          phi_pass<4>(base + own_off, own_bytes, 2 * kPanel, 2, row0, tail ? qt : qf,
                      tail ? kt : kf, factored, ident, tt, kXformThreads);
        fence_proxy_async_smem();
        named_bar_sync(kBarXform, kXformThreads);
        if (rf) return false;
        if (tt == 0) {
          const uint32_t pb = bar((g == 0 ? kPhi0 : kPhiB0) + s);
          if (kPair) {
            const uint32_t src = sb + s * kStage + kOffQ + g * kPanel + own_off;
            const uint32_t dst = map_to_rank(src, peer);
            const uint32_t pbar = map_to_rank(pb, peer);
            bulk_copy_to_peer(dst, src, kPanel / 2, pbar);                            // q rows
            bulk_copy_to_peer(dst + 2 * kPanel, src + 2 * kPanel, kPanel / 2, pbar);  // k rows
            // completes when the peer's rows of this half have arrived here
            mbar_arrive_expect_tx(pb, kPanel);
          } else {
            mbar_arrive(pb);
          }
        }
      }
      return true;
    };
    auto weight_k = [&](int c) -> bool {
      const int s = c & 1;
      check(mbar_wait(bar(kAFull0 + s), (c >> 1) & 1));   // the score MMA has read phi(K)
      const float *wk = c == nchunks - 1 ? kt : kf;
      if (!rf)
        tile_pass<4>(sm + s * kStage + kOffK, 2 * kPanel, 2 * kPanel, 1, tt, kXformThreads,
                     [wk](uint32_t w, uint32_t o) {
                       const float f = wk[(o & (kPanel - 1)) >> 7];
                       return mul_bf16x2(w, pack_bf16(f, f));
                     });
      fence_proxy_async_smem();
      named_bar_sync(kBarXform, kXformThreads);
      if (rf) return false;
      if (tt == 0) mbar_arrive(bar(kKsDone));
      return true;
    };
    if (nchunks > 0 && transform(0)) {
      for (int c = 0; c < nchunks; ++c) {
        if (!factored && !weight_k(c)) break;   // the factored decay needs no second pass
        if (c + 1 < nchunks && !transform(c + 1)) break;
      }
    }
  } else if (warp < 12) {
    // ------------------------------------------------ masked score tile
    const int wq = warp - 8;          // TMEM lane quarter and row block
    const int t = wq * 32 + lane;     // query row inside the chunk
    const uint32_t lane_field = static_cast<uint32_t>(wq * 32) << 16;
    volatile int &rf = role_fail[1];
    for (int c = 0; c < nchunks; ++c) {
      const int b = c & 1;
      bool okw = !*abort_flag && mbar_wait(bar(kAFull0 + b), (c >> 1) & 1);
      okw = okw && (c == 0 || mbar_wait(bar(kOvDone), (c - 1) & 1));   // O_in(c-1) read the tile
      if (!okw) {
        rf = 1;
        fail();
      }
      tc_fence_after();
      // only blocks at or below the diagonal change; the others stay zero
      for (int bk = 0; !rf && bk <= wq; ++bk) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(tmem + lane_field + kTmA + b * 128 + bk * 32, r);
        tmem_wait_ld();
        uint32_t pk[16];
        if (factored) {
          // the MMA already produced lambda^(t-s) phi(q).phi(k): only mask s > t
          if (bk < wq) {
#pragma unroll
            for (int i = 0; i < 16; ++i)
              pk[i] = pack_bf16(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i)
              pk[i] = pack_bf16(2 * i <= lane ? __uint_as_float(r[2 * i]) : 0.f,
                                2 * i + 1 <= lane ? __uint_as_float(r[2 * i + 1]) : 0.f);
          }
        } else if (bk < wq) {
          // left of the diagonal: lambda^(t-s) = lambda^(t-s_last) lambda^(31-j)
          const float g = pw[t - (bk * 32 + 31)];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            pk[i] = pack_bf16(__uint_as_float(r[2 * i]) * (g * pw[31 - 2 * i]),
                              __uint_as_float(r[2 * i + 1]) * (g * pw[30 - 2 * i]));
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int j = 2 * i;
            const float f0 = j <= lane ? pw[max(lane - j, 0)] : 0.f;
            const float f1 = j + 1 <= lane ? pw[max(lane - j - 1, 0)] : 0.f;
            pk[i] = pack_bf16(__uint_as_float(r[j]) * f0, __uint_as_float(r[j + 1]) * f1);
          }
        }
        uint8_t *pa = sm + kOffA + (bk >> 1) * kPanel;
#pragma unroll
        for (int i = 0; i < 4; ++i)
          *reinterpret_cast<uint4 *>(pa + sw128_offset(t, (bk & 1) * 64 + i * 16)) =
              make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
      }
      tc_fence_before();
      fence_proxy_async_smem();
      named_bar_sync(kBarEpiA, 128);
      if (rf) break;
      if (t == 0) {
        mbar_arrive(bar(kAFree0 + b));
        mbar_arrive(bar(kAbfFull));
      }
    }
  } else {
    // ---------------------------------------------- state update and output
    const int wq = warp - 12;
    const int r = wq * 32 + lane;     // d_k row (state) and query row (output)
    const uint32_t lane_field = static_cast<uint32_t>(wq * 32) << 16;
    volatile int &rf = role_fail[2];
    for (int c = 0; c < nchunks; ++c) {
      const int Cv = c == nchunks - 1 ? Ct : C;
      const bool last = c == nchunks - 1;
      // -- state after the chunk (needs this chunk's state MMA, and O_x done
      //    reading the previous bf16 state operand)
      bool okw = !*abort_flag && mbar_wait(bar(kDsDone), c & 1) && mbar_wait(bar(kOxDone), c & 1);
      if (!okw) {
        rf = 1;
        fail();
      }
      tc_fence_after();
      if (!rf) {
        uint32_t zz[2];
        tmem_ld_32x32b_x2(tmem + lane_field + kTmS + 64, zz);   // z, junk
        const float gnext = last ? 1.f : pw[c + 1 == nchunks - 1 ? Ct : C];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t sv[32];
          tmem_ld_32x32b_x32(tmem + lane_field + kTmS + half * 32, sv);
          tmem_wait_ld();
          if (last) {
            if (S_final && (!kDk64 || r < dk)) {
              float4 *dst = reinterpret_cast<float4 *>(
                  S_final + (static_cast<long>(pair) * dk + r) * DV + j0 + half * 32);
#pragma unroll
              for (int i = 0; i < 8; ++i)
                dst[i] = make_float4(__uint_as_float(sv[4 * i]), __uint_as_float(sv[4 * i + 1]),
                                     __uint_as_float(sv[4 * i + 2]), __uint_as_float(sv[4 * i + 3]));
            }
          } else {
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              pk[i] = pack_bf16(__uint_as_float(sv[2 * i]), __uint_as_float(sv[2 * i + 1]));
#pragma unroll
            for (int i = 0; i < 4; ++i)
              *reinterpret_cast<uint4 *>(sm + kOffS + sw128_offset(r, half * 64 + i * 16)) =
                  make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
#pragma unroll
            for (int i = 0; i < 32; ++i) sv[i] = __float_as_uint(__uint_as_float(sv[i]) * gnext);
            tmem_st_32x32b_x32(tmem + lane_field + kTmS + half * 32, sv);
          }
        }
        const float zc = __uint_as_float(zz[0]);
        if (last) {
          if (z_final && j0 == 0 && (!kDk64 || r < dk)) z_final[static_cast<long>(pair) * dk + r] = zc;
        } else {
          // z (decayed) back into column 64; the other side columns restart at 0
          uint32_t zcol[16];
          zcol[0] = __float_as_uint(zc * gnext);
#pragma unroll
          for (int i = 1; i < 16; ++i) zcol[i] = 0u;
          tmem_st_32x32b_x16(tmem + lane_field + kTmS + 64, zcol);
          tmem_wait_st();
          // z as a bf16 hi/lo pair in columns 1-2 of the shared atom (row = d_k)
          const __nv_bfloat16 zh = __float2bfloat16_rn(zc);
          const __nv_bfloat16 zl = __float2bfloat16_rn(zc - __bfloat162float(zh));
          *reinterpret_cast<__nv_bfloat16 *>(sm + kOffX + sw128_offset(r, 2)) = zh;
          *reinterpret_cast<__nv_bfloat16 *>(sm + kOffX + sw128_offset(r, 4)) = zl;
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      named_bar_sync(kBarOut, 128);
      if (rf) break;
      if (r == 0) mbar_arrive(bar(kStateDone));
      // -- y for the chunk's rows
      okw = !*abort_flag && mbar_wait(bar(kOvDone), c & 1);
      if (!okw) {
        rf = 1;
        fail();
      }
      tc_fence_after();
      if (!rf) {
        uint32_t rs[2], qz[2];
        tmem_ld_32x32b_x2(tmem + lane_field + kTmOV + 64, rs);   // row sum, junk
        tmem_ld_32x32b_x2(tmem + lane_field + kTmOX + 65, qz);   // qz hi, lo parts
        tmem_wait_ld();
        // weight of the carried state: lambda^(t+1), or lambda^Cv when phi(q)
        // already carries lambda^(t+1-Cv)
        const float g = factored ? pw[Cv] : pw[r + 1];
        const float inv =
            1.f / (__uint_as_float(rs[0]) + g * (__uint_as_float(qz[0]) + __uint_as_float(qz[1])) +
                   eps);
        const long row = static_cast<long>(c) * C + r;
        uint4 *dst = reinterpret_cast<uint4 *>(out + (static_cast<long>(pair) * N + row) * DV + j0);
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
          uint32_t oi[16], ox[16];
          tmem_ld_32x32b_x16(tmem + lane_field + kTmOV + qq * 16, oi);
          tmem_ld_32x32b_x16(tmem + lane_field + kTmOX + qq * 16, ox);
          tmem_wait_ld();
          uint32_t pk[8];
#pragma unroll
          for (int i = 0; i < 8; ++i)
            pk[i] = pack_bf16(fmaf(g, __uint_as_float(ox[2 * i]), __uint_as_float(oi[2 * i])) * inv,
                              fmaf(g, __uint_as_float(ox[2 * i + 1]), __uint_as_float(oi[2 * i + 1])) *
                                  inv);
          if (r < Cv) {
            dst[qq * 2] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            dst[qq * 2 + 1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
          }
        }
      }
      tc_fence_before();
      named_bar_sync(kBarOut, 128);
      if (rf) break;
      if (r == 0) mbar_arrive(bar(kOutDone));
    }
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmCols);
  }
  // no remote arrival or copy may target a CTA that has exited
  if (kPair) cluster_sync_all();
}

}  // namespace tc
}  // namespace linattn
