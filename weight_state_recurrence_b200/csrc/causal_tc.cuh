// Chunked causal forward on the 5th-generation tensor cores (bf16 operands,
// fp32 accumulators in TMEM), d_k = 128, dv sliced 64 columns per CTA.
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
//   S     <- lambda^Cv S + phi(K)^T (Lk V),   Lk = diag(lambda^(Cv-1-t))
//   z     <- lambda^Cv z + phi(K)^T (Lk 1)
//
// Every product is a tcgen05.mma chain issued by one thread (M = 128):
//   A     N=128 K=128(d_k)  phi(Q) K-major x phi(K) K-major   -> TMEM (2 buffers)
//   O_in  N=64  K=128(s)    A bf16 K-major x V MN-major
//   rs    N=16  K=128(s)    A bf16 x W (row 0 = ones)
//   O_x   N=64  K=128(d_k)  phi(Q) x S bf16 MN-major
//   qz    N=16  K=128(d_k)  phi(Q) x Z (rows: z_hi, z_lo)
//   S     N=64  K=128(t)    phi(K)^T MN-major x Lk V MN-major, accumulated onto
//                           the fp32 state that stays in TMEM
//   dz    N=16  K=128(t)    phi(K)^T x W (rows 1, 2: hi / lo of lambda^(Cv-1-t))
// The fp32 state S never leaves the tensor memory between chunks: after each
// chunk one warpgroup reads it, emits it as the bf16 operand of the next
// chunk's O_x, and writes it back multiplied by lambda^Cv so that the next
// S MMA accumulates onto the decayed state.  The denominator sums exactly
// the bf16-rounded weights the numerator uses (rs comes from the same bf16 A
// tile), so y stays a normalised average of values.
//
// Warp roles (512 threads):
//   warp 0      TMA producer: q, k, v tiles of a chunk into a 2-stage ring
//   warp 1      TMEM owner and the single MMA-issuing thread
//   warps 2-7   phi applied in place to q and k tiles (packed bf16x2), and
//               the in-place decay weighting of V for the state update
//   warps 8-11  masked, decayed score tile: TMEM -> registers -> bf16 SMEM
//   warps 12-15 output (y = numerator / denominator, stored to HBM) and the
//               state update
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
constexpr int NT = 512;

constexpr int kXformThreads = 192;  // warps 2-7
constexpr int kBarXform = 1, kBarEpiA = 2, kBarOut = 3;  // named barrier ids

// ---- shared memory (offsets from a 1024-byte aligned base)
constexpr uint32_t kPanel = C * 128;            // 128 rows x 128 bytes
constexpr uint32_t kOffQ = 0;                   // per stage: phi(Q), 2 panels (d_k 0-63, 64-127)
constexpr uint32_t kOffK = 2 * kPanel;          //            phi(K), 2 panels
constexpr uint32_t kOffV = 4 * kPanel;          //            V slice, 1 panel
constexpr uint32_t kStage = 5 * kPanel;         // 80 KB
constexpr uint32_t kOffA = 2 * kStage;          // bf16 score tile, 2 panels (keys 0-63, 64-127)
constexpr uint32_t kOffS = kOffA + 2 * kPanel;  // bf16 S slice operand, 1 panel
constexpr uint32_t kOffZ = kOffS + kPanel;      // [z_hi; z_lo; 0 ...] 16 x 128, 2 panels of 2 KB
constexpr uint32_t kOffW = kOffZ + 4096;        // [1; w_hi; w_lo; 0 ...] for full chunks
constexpr uint32_t kOffWt = kOffW + 4096;       // same for the last (ragged) chunk
constexpr uint32_t kOffMisc = kOffWt + 4096;
constexpr uint32_t kMiscBytes = 2560;
constexpr uint32_t kSmemBytes = kOffMisc + kMiscBytes + 1024;  // + alignment slack
constexpr uint32_t kStageTxBytes = 5 * kPanel;

// ---- barriers (8 bytes each, at kOffMisc)
enum Bar {
  kFull0 = 0, kFull1, kPhi0, kPhi1, kFree0, kFree1, kAFull0, kAFull1, kAFree0, kAFree1,
  kAbfFull, kOvDone, kOxDone, kVsDone, kDsDone, kStateDone, kOutDone, kFinal, kNumBars
};
constexpr uint32_t kMiscTmem = 160, kMiscAbort = 164, kMiscConsumed = 168;
constexpr uint32_t kMiscPw = 192;                    // lambda^i, i = 0..C      (132 floats)
constexpr uint32_t kMiscQs = kMiscPw + 132 * 4;      // lambda^(t+1)           (128 floats)
constexpr uint32_t kMiscVf = kMiscQs + 128 * 4;      // lambda^(C-1-t)         (128 floats)
constexpr uint32_t kMiscVt = kMiscVf + 128 * 4;      // lambda^(Ct-1-t), 0 past Ct
static_assert(kMiscVt + 128 * 4 <= kMiscBytes, "misc region overflow");

// ---- tensor memory columns (fp32, lane = row)
constexpr uint32_t kTmA = 0;      // two 128-column score buffers
constexpr uint32_t kTmOI = 256;   // O_in  (64)
constexpr uint32_t kTmOX = 320;   // O_x   (64)
constexpr uint32_t kTmS = 384;    // state (64), lane = d_k row
constexpr uint32_t kTmRS = 448;   // rs    (16)
constexpr uint32_t kTmQZ = 464;   // qz    (16)
constexpr uint32_t kTmDZ = 480;   // dz    (16), lane = d_k row
constexpr uint32_t kTmCols = 512;

constexpr uint32_t kIdA = idesc_bf16(128, 128, 0, 0);
constexpr uint32_t kIdN64 = idesc_bf16(128, 64, 0, 1);    // K-major A, MN-major B
constexpr uint32_t kIdN16 = idesc_bf16(128, 16, 0, 0);    // K-major A, K-major B
constexpr uint32_t kIdS = idesc_bf16(128, 64, 1, 1);      // MN-major A, MN-major B
constexpr uint32_t kIdDZ = idesc_bf16(128, 16, 1, 0);     // MN-major A, K-major B

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

__global__ void __launch_bounds__(NT, 1)
    causal_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                     const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const float *__restrict__ lam,
                     float eps, __nv_bfloat16 *__restrict__ out, float *__restrict__ S_final,
                     float *__restrict__ z_final, int H, int N, int DV) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                            ~static_cast<uintptr_t>(1023));
  const uint32_t sb = smem_u32(sm);
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int nslices = DV / DVS;
  const int pair = blockIdx.x / nslices;
  const int j0 = (blockIdx.x % nslices) * DVS;
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
  float *qs = reinterpret_cast<float *>(misc + kMiscQs);
  float *vf = reinterpret_cast<float *>(misc + kMiscVf);
  float *vt = reinterpret_cast<float *>(misc + kMiscVt);

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
  __syncthreads();
  if (tid < C) {
    qs[tid] = pw[tid + 1];
    vf[tid] = pw[C - 1 - tid];
    vt[tid] = tid < Ct ? pw[Ct - 1 - tid] : 0.f;
  }
  __syncthreads();
  // constant operand tiles: S = 0, Z = 0, W / Wt = [1; w_hi; w_lo; 0 ...],
  // and the score tile's blocks above the diagonal (always zero)
  for (uint32_t o = tid * 16u; o < kPanel; o += NT * 16u)
    *reinterpret_cast<uint4 *>(sm + kOffS + o) = make_uint4(0, 0, 0, 0);
  for (uint32_t o = tid * 16u; o < 3 * 4096u; o += NT * 16u)
    *reinterpret_cast<uint4 *>(sm + kOffZ + o) = make_uint4(0, 0, 0, 0);
  for (uint32_t o = tid * 16u; o < 2 * kPanel; o += NT * 16u)
    *reinterpret_cast<uint4 *>(sm + kOffA + o) = make_uint4(0, 0, 0, 0);
  __syncthreads();
  if (tid < C) {
    const int t = tid;
    const __nv_bfloat16 one = __float2bfloat16_rn(1.f);
    const float wf = vf[t], wt = vt[t];
    const __nv_bfloat16 fh = __float2bfloat16_rn(wf), th = __float2bfloat16_rn(wt);
    const __nv_bfloat16 fl = __float2bfloat16_rn(wf - __bfloat162float(fh));
    const __nv_bfloat16 tl = __float2bfloat16_rn(wt - __bfloat162float(th));
    __nv_bfloat16 *W = reinterpret_cast<__nv_bfloat16 *>(sm + kOffW);
    __nv_bfloat16 *Wt = reinterpret_cast<__nv_bfloat16 *>(sm + kOffWt);
    W[kmajor_off(0, t, 2048) / 2] = one;
    W[kmajor_off(1, t, 2048) / 2] = fh;
    W[kmajor_off(2, t, 2048) / 2] = fl;
    Wt[kmajor_off(0, t, 2048) / 2] = one;
    Wt[kmajor_off(1, t, 2048) / 2] = th;
    Wt[kmajor_off(2, t, 2048) / 2] = tl;
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  auto fail = [&]() { *abort_flag = 1; };

  if (warp == 0) {
    // ------------------------------------------------------- TMA producer
    int issued = 0;
    if (lane == 0) {
      for (int c = 0; c < nchunks && !*abort_flag; ++c) {
        const int s = c & 1;
        if (c >= 2 && !mbar_wait(bar(kFree0 + s), ((c - 2) >> 1) & 1)) {
          fail();
          break;
        }
        const uint32_t base = sb + s * kStage;
        const uint32_t b = bar(kFull0 + s);
        mbar_arrive_expect_tx(b, kStageTxBytes);
        tma_load_3d(base + kOffQ, &tm_q, b, 0, c * C, pair);
        tma_load_3d(base + kOffQ + kPanel, &tm_q, b, 64, c * C, pair);
        tma_load_3d(base + kOffK, &tm_k, b, 0, c * C, pair);
        tma_load_3d(base + kOffK + kPanel, &tm_k, b, 64, c * C, pair);
        tma_load_3d(base + kOffV, &tm_v, b, j0, c * C, pair);
        issued = c + 1;
      }
      if (*abort_flag) {
        // let every copy this thread started land before the CTA exits
        for (int c = *consumed; c < issued; ++c) mbar_wait(bar(kFull0 + (c & 1)), (c >> 1) & 1);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      auto mma_scores = [&](int c) -> bool {
        const int s = c & 1;
        if (!mbar_wait(bar(kPhi0 + s), (c >> 1) & 1)) return false;
        if (c >= 2 && !mbar_wait(bar(kAFree0 + s), ((c - 2) >> 1) & 1)) return false;
        tc_fence_after();
        const uint32_t st = sb + s * kStage;
#pragma unroll
        for (int ks = 0; ks < DK / 16; ++ks) {
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
        const uint32_t w = sb + (c == nchunks - 1 ? kOffWt : kOffW);
        if (*abort_flag) break;
        if (c + 1 < nchunks && !(ok = mma_scores(c + 1))) break;
        // O_x = phi(Q) S, qz = phi(Q) z   (state of the previous chunk)
        if (c >= 1 && (!mbar_wait(bar(kStateDone), (c - 1) & 1) ||
                       !mbar_wait(bar(kOutDone), (c - 1) & 1))) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < DK / 16; ++ks) {
          const uint32_t off = (ks >> 2) * kPanel + (ks & 3) * 32;
          const uint64_t a = sdesc_sw128(st + kOffQ + off, 16, 1024);
          umma_bf16(tmem + kTmOX, a, sdesc_sw128(sb + kOffS + ks * 2048, kPanel, 1024), kIdN64,
                    ks > 0);
          umma_bf16(tmem + kTmQZ, a,
                    sdesc_sw128(sb + kOffZ + (ks >> 2) * 2048 + (ks & 3) * 32, 16, 1024), kIdN16,
                    ks > 0);
        }
        umma_commit(bar(kOxDone));
        // O_in = A V, rs = A 1
        if (!mbar_wait(bar(kAbfFull), c & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < C / 16; ++ks) {
          const uint64_t a = sdesc_sw128(sb + kOffA + (ks >> 2) * kPanel + (ks & 3) * 32, 16, 1024);
          umma_bf16(tmem + kTmOI, a, sdesc_sw128(st + kOffV + ks * 2048, kPanel, 1024), kIdN64,
                    ks > 0);
          umma_bf16(tmem + kTmRS, a, sdesc_sw128(w + (ks >> 2) * 2048 + (ks & 3) * 32, 16, 1024),
                    kIdN16, ks > 0);
        }
        umma_commit(bar(kOvDone));
        // S += phi(K)^T (Lk V), dz = phi(K)^T (Lk 1)
        if (!mbar_wait(bar(kVsDone), c & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < C / 16; ++ks) {
          const uint64_t a = sdesc_sw128(st + kOffK + ks * 2048, kPanel, 1024);
          umma_bf16(tmem + kTmS, a, sdesc_sw128(st + kOffV + ks * 2048, kPanel, 1024), kIdS,
                    (c > 0 || ks > 0) ? 1u : 0u);
          umma_bf16(tmem + kTmDZ, a, sdesc_sw128(w + (ks >> 2) * 2048 + (ks & 3) * 32, 16, 1024),
                    kIdDZ, ks > 0);
        }
        umma_commit(bar(kDsDone));
        umma_commit(bar(kFree0 + s));
      }
      if (!ok) fail();
      // make sure nothing this thread issued is still running
      umma_commit(bar(kFinal));
      mbar_wait(bar(kFinal), 0);
    }
    __syncwarp();
  } else if (warp < 8) {
    // ------------------------------------------- phi transform, V weighting
    const int tt = tid - 64;
    auto transform = [&](int c) -> bool {
      const int s = c & 1;
      if (!mbar_wait(bar(kFull0 + s), (c >> 1) & 1)) return false;
      if (tt == 0) *consumed = c + 1;
      uint8_t *p = sm + s * kStage + kOffQ;  // q and k tiles are adjacent (64 KB)
      for (uint32_t o = tt * 16u; o < 4 * kPanel; o += kXformThreads * 16u) {
        uint4 w = *reinterpret_cast<uint4 *>(p + o);
        w.x = phi_bf16x2(w.x);
        w.y = phi_bf16x2(w.y);
        w.z = phi_bf16x2(w.z);
        w.w = phi_bf16x2(w.w);
        *reinterpret_cast<uint4 *>(p + o) = w;
      }
      fence_proxy_async_smem();
      named_bar_sync(kBarXform, kXformThreads);
      if (tt == 0) mbar_arrive(bar(kPhi0 + s));
      return true;
    };
    auto weight_v = [&](int c) -> bool {
      const int s = c & 1;
      if (!mbar_wait(bar(kOvDone), c & 1)) return false;
      const float *wv = c == nchunks - 1 ? vt : vf;
      uint8_t *p = sm + s * kStage + kOffV;
      for (uint32_t o = tt * 16u; o < kPanel; o += kXformThreads * 16u) {
        const float f = wv[o >> 7];
        const uint32_t f2 = pack_bf16(f, f);
        uint4 w = *reinterpret_cast<uint4 *>(p + o);
        w.x = mul_bf16x2(w.x, f2);
        w.y = mul_bf16x2(w.y, f2);
        w.z = mul_bf16x2(w.z, f2);
        w.w = mul_bf16x2(w.w, f2);
        *reinterpret_cast<uint4 *>(p + o) = w;
      }
      fence_proxy_async_smem();
      named_bar_sync(kBarXform, kXformThreads);
      if (tt == 0) mbar_arrive(bar(kVsDone));
      return true;
    };
    bool ok = nchunks > 0 && transform(0);
    for (int c = 0; ok && c < nchunks; ++c) {
      if (*abort_flag) break;
      if (c + 1 < nchunks && !(ok = transform(c + 1))) break;
      ok = weight_v(c);
    }
    if (!ok) fail();
  } else if (warp < 12) {
    // ------------------------------------------------ masked score tile
    const int wq = warp - 8;          // TMEM lane quarter and row block
    const int t = wq * 32 + lane;     // query row inside the chunk
    const uint32_t lane_field = static_cast<uint32_t>(wq * 32) << 16;
    bool ok = true;
    for (int c = 0; c < nchunks; ++c) {
      const int b = c & 1;
      if (*abort_flag) break;
      if (!mbar_wait(bar(kAFull0 + b), (c >> 1) & 1) ||
          (c >= 1 && !mbar_wait(bar(kOvDone), (c - 1) & 1))) {
        ok = false;
        break;
      }
      tc_fence_after();
      // only blocks at or below the diagonal change; the others stay zero
      for (int blk = 0; blk <= wq; ++blk) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(tmem + lane_field + kTmA + b * 128 + blk * 32, r);
        tmem_wait_ld();
        float f[32];
        if (blk < wq) {
          // whole block left of the diagonal: lambda^(t-s) from the last column back
          float g = pw[t - (blk * 32 + 31)];
#pragma unroll
          for (int j = 31; j >= 0; --j) {
            f[j] = g;
            g *= L;
          }
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) f[j] = j <= lane ? pw[max(lane - j, 0)] : 0.f;
        }
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk[i] = pack_bf16(__uint_as_float(r[2 * i]) * f[2 * i],
                            __uint_as_float(r[2 * i + 1]) * f[2 * i + 1]);
        uint8_t *pa = sm + kOffA + (blk >> 1) * kPanel;
#pragma unroll
        for (int i = 0; i < 4; ++i)
          *reinterpret_cast<uint4 *>(pa + sw128_offset(t, (blk & 1) * 64 + i * 16)) =
              make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
      }
      tc_fence_before();
      fence_proxy_async_smem();
      named_bar_sync(kBarEpiA, 128);
      if (t == 0) {
        mbar_arrive(bar(kAFree0 + b));
        mbar_arrive(bar(kAbfFull));
      }
    }
    if (!ok) fail();
  } else {
    // ---------------------------------------------- output and state update
    const int wq = warp - 12;
    const int r = wq * 32 + lane;     // query row (output) and d_k row (state)
    const uint32_t lane_field = static_cast<uint32_t>(wq * 32) << 16;
    float z_reg = 0.f;
    bool ok = true;
    for (int c = 0; c < nchunks; ++c) {
      if (*abort_flag) break;
      const int Cv = c == nchunks - 1 ? Ct : C;
      // -- y for the chunk's rows
      if (!mbar_wait(bar(kOxDone), c & 1) || !mbar_wait(bar(kOvDone), c & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      {
        uint32_t rs[2], qz[2];
        tmem_ld_32x32b_x2(tmem + lane_field + kTmRS, rs);
        tmem_ld_32x32b_x2(tmem + lane_field + kTmQZ, qz);
        tmem_wait_ld();
        const float g = qs[r];
        const float inv =
            1.f / (__uint_as_float(rs[0]) + g * (__uint_as_float(qz[0]) + __uint_as_float(qz[1])) +
                   eps);
        const long row = static_cast<long>(c) * C + r;
        uint4 *dst = reinterpret_cast<uint4 *>(out + (static_cast<long>(pair) * N + row) * DV + j0);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t oi[32], ox[32];
          tmem_ld_32x32b_x32(tmem + lane_field + kTmOI + half * 32, oi);
          tmem_ld_32x32b_x32(tmem + lane_field + kTmOX + half * 32, ox);
          tmem_wait_ld();
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            pk[i] = pack_bf16(fmaf(g, __uint_as_float(ox[2 * i]), __uint_as_float(oi[2 * i])) * inv,
                              fmaf(g, __uint_as_float(ox[2 * i + 1]), __uint_as_float(oi[2 * i + 1])) *
                                  inv);
          if (r < Cv) {
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[half * 4 + i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
          }
        }
      }
      tc_fence_before();
      named_bar_sync(kBarOut, 128);
      if (r == 0) mbar_arrive(bar(kOutDone));
      // -- state after the chunk
      if (!mbar_wait(bar(kDsDone), c & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const bool last = c == nchunks - 1;
      {
        uint32_t dz[2];
        tmem_ld_32x32b_x2(tmem + lane_field + kTmDZ + 1, dz);
        tmem_wait_ld();
        z_reg = fmaf(pw[Cv], z_reg, __uint_as_float(dz[0]) + __uint_as_float(dz[1]));
        const float gnext = last ? 1.f : pw[c + 1 == nchunks - 1 ? Ct : C];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t sv[32];
          tmem_ld_32x32b_x32(tmem + lane_field + kTmS + half * 32, sv);
          tmem_wait_ld();
          if (last) {
            if (S_final) {
              float4 *dst = reinterpret_cast<float4 *>(
                  S_final + (static_cast<long>(pair) * DK + r) * DV + j0 + half * 32);
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
        if (last) {
          if (z_final && j0 == 0) z_final[static_cast<long>(pair) * DK + r] = z_reg;
        } else {
          tmem_wait_st();
          const __nv_bfloat16 zh = __float2bfloat16_rn(z_reg);
          const __nv_bfloat16 zl = __float2bfloat16_rn(z_reg - __bfloat162float(zh));
          __nv_bfloat16 *Z = reinterpret_cast<__nv_bfloat16 *>(sm + kOffZ);
          Z[kmajor_off(0, r, 2048) / 2] = zh;
          Z[kmajor_off(1, r, 2048) / 2] = zl;
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      named_bar_sync(kBarOut, 128);
      if (r == 0) mbar_arrive(bar(kStateDone));
    }
    if (!ok) fail();
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmCols);
  }
}

}  // namespace tc
}  // namespace linattn
