// Backward of the chunked causal forward on the 5th-generation tensor cores:
// bf16 operands, fp32 accumulators in TMEM, d_k = d_v = 128, chunks of C = 128
// tokens.  Three passes, each one CTA per (b, h) walking the chunks:
//
// The loss is L = sum_i dy_i . y_i with y_i = num_i / den_i (fast-weight
// article §2.1, §3.2, §4.2: S_i = lambda S_(i-1) + phi(k_i) v_i^T, z likewise,
// num_i = phi(q_i)^T S_i, den_i = phi(q_i)^T z_i + eps).  Per token
//   dnum_i = dy_i / den_i,   dden_i = -(dy_i . num_i) / den_i^2 = -dnum_i . y_i
// (formed here from the bf16 dnum_i the products use, so that the key weight
// dnum_i . v_j + dden_i = dnum_i . (v_j - y_i) stays exact where it cancels)
// and the three gradients are linear attentions of their own:
//   dphi(q_i) = S_i dnum_i + z_i dden_i                       (causal, keys j <= i)
//   dphi(k_j) = sum_{i>=j} lambda^(i-j) phi(q_i) (dnum_i . v_j + dden_i)
//   dv_j      = sum_{i>=j} lambda^(i-j) (phi(q_i) . phi(k_j)) dnum_i
// (the last two anti-causal), dq = dphi(q) phi'(q), dk = dphi(k) phi'(k) with
// phi'(x) = 1 for x > 0 and e^x = phi(x) otherwise, i.e. min(phi(x), 1).
//
// Per chunk (t, s local token indices, Q = phi(q) rows, K = phi(k) rows,
// M[t][s] = lambda^(t-s) for s <= t, P = Q K^T, w_t = dnum_t):
//   pass F (chunks in order; state S, z at the chunk start):
//     A = P o M,  num = diag(lambda^(t+1)) Q S + A V,  den = lambda^(t+1) Q z + A 1 + eps
//     W = w V^T,  B = (W + dden 1^T) o M
//     dphi(Q) = diag(lambda^(t+1)) (w S^T + dden z^T) + B K
//     S <- lambda^C S + (Lk K)^T V,  Lk = diag(lambda^(C-1-s))     (z on CUDA cores)
//   pass R (chunks in reverse; R, r = the adjoint of every later token,
//   R = sum_{later t} lambda^(t - chunk end) Q_t w_t^T):
//     dv      = A^T w + Lk K R
//     dphi(K) = B^T Q + Lk (V R^T + 1 r^T)
//     R <- lambda^C R + (Lq Q)^T w,  Lq = diag(lambda^(t+1))           (r likewise)
//   The per-token den_t and dden_t pass from F to L and R through a stash:
//   two floats per token at a caller-given stride (a workspace, or the first
//   8 bytes of the token's dk row, which R overwrites afterwards; then L must
//   finish before R starts).
//
// dlambda = sum_{s<t} (t-s) lambda^(t-s-1) (Q_t . K_s)(w_t . v_s + dden_t)
// is split by where the pair (t, s) lies.  Both in the chunk: the tile
// A' = P o M', M'[t][s] = (t-s) lambda^(t-s-1), against W + dden (pass F).
// Key before the chunk: the chunk-start state enters token t as
// lambda^(t+1) S, whose lambda-derivative is (t+1) lambda^t S + lambda^(t+1) S'
// with S' = dS/dlambda.  The first part is (t+1) lambda^t Q_t . (S w_t + z dden_t),
// read off pass F's own S w product; the second needs S' and is pass L
// (dlambda only):
//     Ms = (Lq Q)^T w,   dlambda += <S', Ms> + sum_t dden_t lambda^(t+1) Q_t . z'
//     S' <- lambda^C S' + C lambda^(C-1) S + (Lk' K)^T V,  Lk' = diag((C-1-s) lambda^(C-2-s))
// Every power is a table entry lambda^m or m lambda^(m-1) formed directly, so
// lambda = 0 and lambda = 1 need no special case.
//
// Each pass is four warpgroups (512 threads) that own the same rows (thread =
// row of the token tile or of the state, TMEM lane = row) and split each row's
// 128 columns in quarters; row sums meet through shared memory at the block
// barriers.  Thread 0 issues the MMAs in program order: the role split and the
// deep pipelines of the forward are not used here.  Waits are bounded: thread
// 0 polls the copy barriers and every thread the MMA barriers; a wait that
// runs out sets a shared flag, and every thread leaves the chunk loop together
// at the next block barrier.
#pragma once
#include "common.cuh"
#include "sm100.cuh"
#include "causal_tc.cuh"

namespace linattn {
namespace btc {

using tc::mul_bf16x2;
using tc::pack_bf16;
using tc::phi_bf16x2;

constexpr int C = 128;     // tokens per chunk
constexpr int D = 128;     // d_k = d_v
constexpr uint32_t kPanel = 128u * 128u;   // 128 rows x 128 bytes (64 bf16)
constexpr uint32_t kTile = 2u * kPanel;    // 128 x 128 bf16 in two 64-column panels

// byte offset of 16-byte chunk j (0..15) of row r in a tile (128-byte swizzle)
__device__ __forceinline__ uint32_t toff(uint32_t r, uint32_t j) {
  return (j >> 3) * kPanel + sw128_offset(r, (j & 7u) * 16u);
}
__device__ __forceinline__ float blo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bhi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Operand descriptors.  K-major: rows are M (or N), K runs along the row
// (across the two panels).  MN-major: rows are K, M (or N) runs along the row.
__device__ __forceinline__ uint64_t kdesc(uint32_t a) { return sdesc_sw128(a, 16, 1024); }
__device__ __forceinline__ uint64_t mdesc(uint32_t a) { return sdesc_sw128(a, kPanel, 1024); }
__device__ __forceinline__ uint64_t kstep(int ks) {
  return static_cast<uint64_t>((ks >> 2) * kPanel + (ks & 3) * 32) >> 4;
}
__device__ __forceinline__ uint64_t mstep(int ks) { return static_cast<uint64_t>(ks * 2048) >> 4; }

constexpr uint32_t kIdKK = idesc_bf16(128, 128, 0, 0);
constexpr uint32_t kIdKM = idesc_bf16(128, 128, 0, 1);
constexpr uint32_t kIdMM = idesc_bf16(128, 128, 1, 1);

// D (+)= A B, K = 128 in 8 steps, both operands in shared memory
__device__ __forceinline__ void mma_ss(uint32_t d, uint64_t a, bool a_mn, uint64_t b, bool b_mn,
                                       bool acc) {
  const uint32_t id = a_mn ? kIdMM : (b_mn ? kIdKM : kIdKK);
#pragma unroll
  for (int ks = 0; ks < 8; ++ks)
    umma_bf16(d, a + (a_mn ? mstep(ks) : kstep(ks)), b + (b_mn ? mstep(ks) : kstep(ks)), id,
              (acc || ks > 0) ? 1u : 0u);
}
// D (+)= A B, A in tensor memory (bf16 pairs, lane = row), B in shared memory
__device__ __forceinline__ void mma_ts(uint32_t d, uint32_t a, uint64_t b, bool b_mn, bool acc) {
  const uint32_t id = b_mn ? kIdKM : kIdKK;
#pragma unroll
  for (int ks = 0; ks < 8; ++ks)
    umma_bf16_ts(d, a + ks * 8, b + (b_mn ? mstep(ks) : kstep(ks)), id,
                 (acc || ks > 0) ? 1u : 0u);
}

// The row helpers below work on this thread's part h of row r when the row's
// 128 columns are cut into P parts (the passes use P = 4, one per
// warpgroup): 16-byte chunks [h 16/P, (h + 1) 16/P).

// The half row through the feature map in place (nothing with `ident`);
// returns phi(row) . vec over the half (fp32) when vec is given and adds the
// half row's sum to *sum when sum is given.
template <int P>
__device__ __forceinline__ float phi_row(uint8_t *tile, int r, int h, bool ident, const float *vec,
                                         float *sum = nullptr) {
  constexpr int CH = 16 / P;
  float acc = 0.f, rs = 0.f;
#pragma unroll 4
  for (int j = CH * h; j < CH * h + CH; ++j) {
    uint4 *p = reinterpret_cast<uint4 *>(tile + toff(r, j));
    uint4 w = *p;
    if (!ident) {
      w.x = phi_bf16x2(w.x);
      w.y = phi_bf16x2(w.y);
      w.z = phi_bf16x2(w.z);
      w.w = phi_bf16x2(w.w);
      *p = w;
    }
    const uint32_t e[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      if (vec) acc += blo(e[m]) * vec[8 * j + 2 * m] + bhi(e[m]) * vec[8 * j + 2 * m + 1];
      rs += blo(e[m]) + bhi(e[m]);
    }
  }
  if (sum) *sum += rs;
  return acc;
}

// elu(x) = phi(x) - 1, in fp32 (e^x - 1 from the fast exponential: its
// absolute error is far below the bf16 rounding that follows)
__device__ __forceinline__ float elu_f32(float x) { return x > 0.f ? x : __expf(x) - 1.f; }

// The half row of a bf16 k tile -> elu(k) in place (nothing with `ident`).
// The key side of every product is carried as elu(k) = phi(k) - 1 plus exact
// rank-one terms for the 1: for small k, phi(k) is 1 plus a small part that
// bf16 near 1 would resolve to only ~2^-8, and the gradient of q lives in
// that part.
template <int P>
__device__ __forceinline__ void elu_row(uint8_t *tile, int r, int h, bool ident) {
  constexpr int CH = 16 / P;
  if (ident) return;
#pragma unroll 4
  for (int j = CH * h; j < CH * h + CH; ++j) {
    uint4 *p = reinterpret_cast<uint4 *>(tile + toff(r, j));
    uint4 w = *p;
    w.x = pack_bf16(elu_f32(blo(w.x)), elu_f32(bhi(w.x)));
    w.y = pack_bf16(elu_f32(blo(w.y)), elu_f32(bhi(w.y)));
    w.z = pack_bf16(elu_f32(blo(w.z)), elu_f32(bhi(w.z)));
    w.w = pack_bf16(elu_f32(blo(w.w)), elu_f32(bhi(w.w)));
    *p = w;
  }
}

// dst half row = src half row * f (bf16 product), dst may be src
template <int P>
__device__ __forceinline__ void scale_row(uint8_t *dst, const uint8_t *src, int r, int h, float f) {
  constexpr int CH = 16 / P;
  const uint32_t f2 = pack_bf16(f, f);
#pragma unroll 4
  for (int j = CH * h; j < CH * h + CH; ++j) {
    uint4 w = *reinterpret_cast<const uint4 *>(src + toff(r, j));
    w.x = mul_bf16x2(w.x, f2);
    w.y = mul_bf16x2(w.y, f2);
    w.z = mul_bf16x2(w.z, f2);
    w.w = mul_bf16x2(w.w, f2);
    *reinterpret_cast<uint4 *>(dst + toff(r, j)) = w;
  }
}

// The half row of dy -> dnum = dy * inv in place (fp32 product, one rounding)
template <int P>
__device__ __forceinline__ void dnum_row(uint8_t *tile, int r, int h, float inv) {
  constexpr int CH = 16 / P;
#pragma unroll 4
  for (int j = CH * h; j < CH * h + CH; ++j) {
    uint4 *p = reinterpret_cast<uint4 *>(tile + toff(r, j));
    uint4 g = *p;
    g.x = pack_bf16(blo(g.x) * inv, bhi(g.x) * inv);
    g.y = pack_bf16(blo(g.y) * inv, bhi(g.y) * inv);
    g.z = pack_bf16(blo(g.z) * inv, bhi(g.z) * inv);
    g.w = pack_bf16(blo(g.w) * inv, bhi(g.w) * inv);
    *p = g;
  }
}

// Column sums of one or two bf16 tiles over all 128 rows, each optionally
// weighted per row, by all T threads of the block together; thread k < 128
// receives the sums of column k in sa and sb.  Thread t reads 16-byte chunk
// t % 16 of rows t / 16 + (T / 16) m; partial sums meet through `scratch`
// (2 x T/32 x 128 floats, in no live tile).  Holds two block barriers: every
// thread calls it.
template <int T>
__device__ __forceinline__ void col_sums(const uint8_t *ta, const float *wa, const uint8_t *tb,
                                         const float *wb, float *scratch, float &sa, float &sb) {
  constexpr int RG = T / 16, NW = T / 32;   // row groups, warps
  const int t = threadIdx.x, j = t & 15, g = t >> 4, lane = t & 31, w = t >> 5;
  float a[8], b[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) a[e] = b[e] = 0.f;
#pragma unroll
  for (int m = 0; m < 128 / RG; ++m) {
    const int r = g + RG * m;
    const uint4 x = *reinterpret_cast<const uint4 *>(ta + toff(r, j));
    const float fa = wa ? wa[r] : 1.f;
    const uint32_t xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      a[2 * u] += blo(xs[u]) * fa;
      a[2 * u + 1] += bhi(xs[u]) * fa;
    }
    if (tb) {
      const uint4 y = *reinterpret_cast<const uint4 *>(tb + toff(r, j));
      const float fb = wb ? wb[r] : 1.f;
      const uint32_t ys[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        b[2 * u] += blo(ys[u]) * fb;
        b[2 * u + 1] += bhi(ys[u]) * fb;
      }
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    a[e] += __shfl_xor_sync(0xffffffffu, a[e], 16);
    b[e] += __shfl_xor_sync(0xffffffffu, b[e], 16);
  }
  if (lane < 16)
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      scratch[w * 128 + 8 * j + e] = a[e];
      scratch[NW * 128 + w * 128 + 8 * j + e] = b[e];
    }
  __syncthreads();
  if (t < 128) {
    float x = 0.f, y = 0.f;
#pragma unroll
    for (int k = 0; k < NW; ++k) {
      x += scratch[k * 128 + t];
      y += scratch[NW * 128 + k * 128 + t];
    }
    sa = x;
    sb = y;
  }
  __syncthreads();
}

// Masked power tables with an offset, so that a masked decay factor is one
// load: lower[127 - t + s] = lambda^(t-s) for s <= t, else 0 (and likewise
// (t-s) lambda^(t-s-1) in the derivative table); upper[127 - t + s] =
// lambda^(s-t) for s >= t, else 0.  256 entries each, filled by thread m.
__device__ __forceinline__ void fill_masked_tables(float L, int m, float *lower, float *dlower,
                                                   float *upper) {
  if (m >= 256) return;
  const int x = 127 - m;   // t - s for lower, -(s - t) for upper
  if (lower) lower[m] = x >= 0 ? pow_int(L, x) : 0.f;
  if (dlower) dlower[m] = x >= 1 ? static_cast<float>(x) * pow_int(L, x - 1) : 0.f;
  if (upper) upper[m] = x <= 0 ? pow_int(L, -x) : 0.f;
}

// The half row r of the fp32 state in TMEM (this warp's lanes; t already
// holds the lane offset) -> bf16 row r of the operand tile, and the state
// multiplied by `f` written back.
template <int P>
__device__ __forceinline__ void state_to_operand(uint32_t t, uint8_t *tile, int r, int h, float f) {
  constexpr int BL = 4 / P;
#pragma unroll 1
  for (int blk = BL * h; blk < BL * h + BL; ++blk) {
    uint32_t v[32];
    tmem_ld_32x32b_x32(t + blk * 32, v);
    tmem_wait_ld();
    uint32_t pk[16];
#pragma unroll
    for (int i = 0; i < 16; ++i)
      pk[i] = pack_bf16(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
#pragma unroll
    for (int m = 0; m < 4; ++m)
      *reinterpret_cast<uint4 *>(tile + toff(r, blk * 4 + m)) =
          make_uint4(pk[4 * m], pk[4 * m + 1], pk[4 * m + 2], pk[4 * m + 3]);
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * f);
    tmem_st_32x32b_x32(t + blk * 32, v);
  }
  tmem_wait_st();
}

// Sum over the block (at most 16 warps; red holds 16 floats).
__device__ __forceinline__ float block_sum(float x, float *red) {
  x = warp_sum(x);
  const int w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  if ((threadIdx.x & 31) == 0) red[w] = x;
  __syncthreads();
  float s = 0.f;
  for (int k = 0; k < nw; ++k) s += red[k];
  __syncthreads();
  return s;
}

// Per-row sums of a row's parts: slot x holds [parts][128] floats.
struct Halves {
  float *base;
  int h, r;
  int parts = 2;
  __device__ __forceinline__ void put(int x, float v) const {
    base[(parts * x + h) * 128 + r] = v;
  }
  __device__ __forceinline__ float get(int x) const {
    float s = 0.f;
    for (int p = 0; p < parts; ++p) s += base[(parts * x + p) * 128 + r];
    return s;
  }
};

// ============================================================== state pass for split F
// Pass F can run as two CTAs per head: chunks [0, H0) and [H0, nch).  The
// second needs the state at token T = H0 C in pass F's elu form (see below):
//   St = sum_{s<T} lambda^(T-1-s) Kt_s v_s^T,  s = sum_{s<T} lambda^(T-1-s) v_s,
//   zt = sum_{s<T} lambda^(T-1-s) Kt_s,        zeta = sum_{s<T} lambda^(T-1-s).
// This pass walks the first H0 chunks of each head once, weighting key row s
// of chunk c by lambda^((H0-1-c) C) lambda^(C-1-s) (a weight relative to T,
// so no decay pass over the accumulator is needed; weights below the bf16
// range are negligible against the others), and writes the state to `mid`:
// per head St [128][128] fp32, then s [128], zt [128], zeta.
constexpr int kMidFloats = D * D + 2 * D + 4;

namespace ps {
// two stages of (k, v) tiles: the copies of chunk c + 2 are issued once chunk c is done
constexpr uint32_t kOffK0 = 0, kOffV0 = kTile, kStage = 2 * kTile, kOffMisc = 2 * kStage;
enum { kFullK0 = 0, kFullV0, kFullK1, kFullV1, kMma, kFinal, kNumBars };
constexpr uint32_t kMiscTmem = 64, kMiscFlag = 68, kMiscPw = 128;
constexpr uint32_t kMiscW = kMiscPw + 132 * 4, kMiscScr = kMiscW + 128 * 4;
constexpr int kNT = 512, kParts = 4;   // four warpgroups, a quarter of each row each
constexpr uint32_t kSmemBytes = kOffMisc + kMiscScr + 2 * (kNT / 32) * 128 * 4;
static_assert(kSmemBytes <= 232448, "exceeds the per-CTA shared memory of sm_100");
}  // namespace ps

__global__ void __launch_bounds__(ps::kNT, 1)
    bwd_tc_s_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                    const float *__restrict__ lam, float *__restrict__ mid, int H, int N, int H0,
                    bool ident) {
  using namespace ps;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *sm = smem_raw;
  const uint32_t sb = smem_u32(sm);
  const int tid = threadIdx.x, warp = tid >> 5;
  if (sb & 1023u) {
    if (tid == 0) atomicOr(&g_status, kStatusWaitTimeout);
    return;
  }
  // pass F (launched next as this pass's programmatic dependent) starts its
  // first halves at once; its second halves wait for this grid
  grid_launch_dependents();
  const long bh = blockIdx.x;
  const int h = static_cast<int>(bh % H);
  const float L = lam ? lam[h] : 1.f;
  uint8_t *misc = sm + kOffMisc;
  auto bar = [&](int i) { return sb + kOffMisc + 8u * static_cast<uint32_t>(i); };
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(misc + kMiscTmem);
  volatile int *flag = reinterpret_cast<volatile int *>(misc + kMiscFlag);
  float *pw = reinterpret_cast<float *>(misc + kMiscPw);   // lambda^m, m = 0..C
  float *wr = reinterpret_cast<float *>(misc + kMiscW);    // this chunk's row weights
  float *scr = reinterpret_cast<float *>(misc + kMiscScr);
  const int hf = tid >> 7, i = tid & 127;
  int issued[4] = {0, 0, 0, 0}, waited[4] = {0, 0, 0, 0};   // per barrier kFullK0..kFullV1
  auto load = [&](int c) {
    const int st = c & 1;
    for (int which = 0; which < 2; ++which) {
      const CUtensorMap *map = which ? &tm_v : &tm_k;
      const int b = 2 * st + which;
      const uint32_t dst = sb + st * kStage + (which ? kOffV0 : kOffK0);
      mbar_arrive_expect_tx(bar(b), kTile);
      tma_load_3d(dst, map, bar(b), 0, c * C, static_cast<int>(bh));
      tma_load_3d(dst + kPanel, map, bar(b), 64, c * C, static_cast<int>(bh));
      if (c + 2 < H0) tma_prefetch_l2_3d(map, 0, (c + 2) * C, static_cast<int>(bh));
      if (c + 2 < H0) tma_prefetch_l2_3d(map, 64, (c + 2) * C, static_cast<int>(bh));
      ++issued[b];
    }
  };
  if (tid == 0) {
    for (int b = 0; b < kNumBars; ++b) mbar_init(bar(b), 1);
    *flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), 128);
    tmem_relinquish();
  }
  if (tid < 128) pw[tid] = pow_int(L, tid);
  if (tid == 0) pw[C] = pow_int(L, C);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lf = static_cast<uint32_t>((warp & 3) * 32) << 16;
  if (tid == 0)
    for (int c = 0; c < min(H0, 2); ++c) load(c);
  auto poll = [&](int b, int parity) {
    if (tid == 0 && !*flag) {
      if (!mbar_wait(bar(b), static_cast<uint32_t>(parity) & 1u)) *flag = 1;
      else if (b <= kFullV1) ++waited[b];
    }
  };
  auto meet = [&]() -> bool {
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    return *flag == 0;
  };
  int mph = 0;
  // every thread waits for the MMA phase itself (see pass F)
  auto mma_wait_all = [&](int b, int &ph) {
    if (!*flag && !mbar_wait(bar(b), static_cast<uint32_t>(ph) & 1u)) *flag = 1;
    ++ph;
    tc_fence_after();
  };
  float geo = 0.f;   // sum_s lambda^(C-1-s)
  for (int m = 0; m < C; ++m) geo += pw[m];
  float zt_acc = 0.f, s_acc = 0.f, zeta = 0.f;   // thread i < 128: column i of zt and s

  for (int c = 0; c < H0; ++c) {
    const int st = c & 1;
    uint8_t *tk = sm + st * kStage + kOffK0, *tv = sm + st * kStage + kOffV0;
    const float tc = pow_int(L, (H0 - 1 - c) * C);   // lambda^((H0-1-c) C)
    if (tid < 128) wr[i] = tc * pw[C - 1 - i];
    poll(2 * st, c >> 1);
    poll(2 * st + 1, c >> 1);
    if (!meet()) break;
    elu_row<kParts>(tk, i, hf, ident);
    scale_row<kParts>(tk, tk, i, hf, wr[i]);
    fence_proxy_async_smem();
    if (!meet()) break;
    if (tid == 0) {
      mma_ss(tmem, mdesc(smem_u32(tk)), true, mdesc(smem_u32(tv)), true, c > 0);   // St += (W Kt)^T V
      umma_commit(bar(kMma));
    }
    {
      float zc = 0.f, sc = 0.f;
      col_sums<kNT>(tk, nullptr, tv, wr, scr, zc, sc);
      if (tid < 128) {
        zt_acc += zc;
        s_acc += sc;
      }
    }
    zeta += tc * geo;
    mma_wait_all(kMma, mph);
    if (tid == 0 && c + 2 < H0) load(c + 2);   // this stage is free
  }
  if (!*flag && H0 > 0) {
    float *m = mid + bh * kMidFloats;
#pragma unroll 1
    for (int blk = hf; blk < hf + 1; ++blk) {
      uint32_t v[32];
      tmem_ld_32x32b_x32(tmem + lf + blk * 32, v);
      tmem_wait_ld();
      float4 *dst = reinterpret_cast<float4 *>(m + i * D + blk * 32);
#pragma unroll
      for (int e = 0; e < 8; ++e)
        dst[e] = make_float4(__uint_as_float(v[4 * e]), __uint_as_float(v[4 * e + 1]),
                             __uint_as_float(v[4 * e + 2]), __uint_as_float(v[4 * e + 3]));
    }
    if (tid < 128) {
      m[D * D + i] = s_acc;
      m[D * D + D + i] = zt_acc;
    }
    if (tid == 0) m[D * D + 2 * D] = zeta;
  }
  if (tid == 0) {
    for (int b = 0; b < 4; ++b)
      for (int n = waited[b]; n < issued[b]; ++n) mbar_wait(bar(b), n & 1);
    umma_commit(bar(kFinal));
    mbar_wait(bar(kFinal), 0);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// ============================================================== pass F
// The key side in the elu form (o = 1; o = 0 and elu(k) -> k with `ident`):
// K = Kt + o 1 1^T with Kt = elu(K), so
//   P = Q Kt^T + o rq 1^T,  rq = Q 1 (row sums of phi(Q))
//   B K = B Kt + o (B 1) 1^T
// and the state S = St + o 1 s^T, z = zt + o zeta 1 with
//   St = sum_s w_s Kt_s v_s^T,  s = sum_s w_s v_s,  zt = sum_s w_s Kt_s,  zeta = sum_s w_s
// (w_s the decay weight of key s), so that
//   Q S = Q St + o rq s^T,   Q z = Q zt + o rq zeta,
//   S w_t + z dden_t = St w_t + zt dden_t + o (s . w_t + zeta dden_t) 1.
// The score weights A = (o rq 1^T + Q Kt^T) o M keep their o rq part exact
// too: its row sum is o rq_t g_t (g_t = sum_{m<=t} lambda^m) and its product
// with V, dotted with w_t, is o rq_t times the masked row sum of W = w V^T;
// only At = (Q Kt^T) o M goes through bf16.
namespace pf {
constexpr uint32_t kOffQ = 0, kOffK = kTile, kOffV = 2 * kTile, kOffG = 3 * kTile,
                   kOffSb = 4 * kTile, kOffAp = 5 * kTile, kOffMisc = 6 * kTile;
enum { kFullQ = 0, kFullK, kFullV, kFullG, kMma, kMma2, kFinal, kNumBars };
constexpr uint32_t kMiscTmem = 64, kMiscFlag = 68, kMiscPw = 128;
constexpr uint32_t kMiscDpw = kMiscPw + 132 * 4, kMiscPwr = kMiscDpw + 132 * 4;
constexpr uint32_t kMiscZ = kMiscPwr + 128 * 4, kMiscS = kMiscZ + 128 * 4;
constexpr uint32_t kMiscGs = kMiscS + 128 * 4, kMiscRed = kMiscGs + 128 * 4;
constexpr uint32_t kMiscLo = kMiscRed + 64, kMiscDlo = kMiscLo + 256 * 4;
constexpr uint32_t kMiscX = kMiscDlo + 256 * 4;
// four warpgroups: thread (h, r) owns the 32 columns [32h, 32h + 32) of row r;
// the row sums of the parts meet in the exchange slots below
constexpr int kNT = 512, kParts = 4;
enum { kXQz = 0, kXRq, kXRs, kXGn, kXSd, kXGw, kXRb, kNumX };
constexpr uint32_t kSmemBytes = kOffMisc + kMiscX + kNumX * kParts * 128 * 4;
static_assert(kSmemBytes <= 232448, "exceeds the per-CTA shared memory of sm_100");
// tensor memory columns
constexpr uint32_t kTmS = 0, kTmT1 = 128, kTmT2 = 256, kTmA = 384, kTmW = 448;
}  // namespace pf

__global__ void __launch_bounds__(pf::kNT, 1)
    bwd_tc_f_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
                    const float *__restrict__ lam, float eps, __nv_bfloat16 *__restrict__ dq,
                    float *__restrict__ stash, long stash_stride, float *__restrict__ dlam,
                    const float *__restrict__ mid, int H0, int H, int N, bool ident) {
  using namespace pf;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *sm = smem_raw;
  const uint32_t sb = smem_u32(sm);
  const int tid = threadIdx.x, warp = tid >> 5;
  if (sb & 1023u) {
    if (tid == 0) atomicOr(&g_status, kStatusWaitTimeout);
    return;
  }
  // H0 > 0: two CTAs per head, chunks [0, H0) and [H0, nch); the second
  // starts from the state the state pass leaves in `mid`
  const int G = H0 > 0 ? 2 : 1;
  const long BH = gridDim.x / G;
  const int half = static_cast<int>(blockIdx.x / BH);
  const long bh = blockIdx.x % BH;
  const int h = static_cast<int>(bh % H);
  const float L = lam ? lam[h] : 1.f;
  const float o = ident ? 0.f : 1.f;
  const int nch = (N + C - 1) / C;
  const int c0 = half ? H0 : 0, c1 = (G == 2 && half == 0) ? H0 : nch;
  uint8_t *misc = sm + kOffMisc;
  auto bar = [&](int i) { return sb + kOffMisc + 8u * static_cast<uint32_t>(i); };
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(misc + kMiscTmem);
  volatile int *flag = reinterpret_cast<volatile int *>(misc + kMiscFlag);
  float *pw = reinterpret_cast<float *>(misc + kMiscPw);     // lambda^m, m = 0..C
  float *dpw = reinterpret_cast<float *>(misc + kMiscDpw);   // m lambda^(m-1)
  float *pwr = reinterpret_cast<float *>(misc + kMiscPwr);   // lambda^(C-1-s)
  float *zt = reinterpret_cast<float *>(misc + kMiscZ);
  float *sv = reinterpret_cast<float *>(misc + kMiscS);
  float *gs = reinterpret_cast<float *>(misc + kMiscGs);     // sum_{m<=t} lambda^m
  float *red = reinterpret_cast<float *>(misc + kMiscRed);
  float *lo = reinterpret_cast<float *>(misc + kMiscLo);     // masked lambda^(t-s), offset
  float *dlo = reinterpret_cast<float *>(misc + kMiscDlo);   // masked (t-s) lambda^(t-s-1)
  const int hf = tid >> 7, i = tid & 127;   // column part, row
  const Halves X{reinterpret_cast<float *>(misc + kMiscX), hf, i, kParts};
  const CUtensorMap *maps[4] = {&tm_q, &tm_k, &tm_v, &tm_g};
  const uint32_t offs[4] = {kOffQ, kOffK, kOffV, kOffG};
  int issued[4] = {0, 0, 0, 0}, waited[4] = {0, 0, 0, 0};   // thread 0: copies per tile
  auto load = [&](int which, int c) {
    const uint32_t b = bar(kFullQ + which);
    mbar_arrive_expect_tx(b, kTile);
    tma_load_3d(sb + offs[which], maps[which], b, 0, c * C, static_cast<int>(bh));
    tma_load_3d(sb + offs[which] + kPanel, maps[which], b, 64, c * C, static_cast<int>(bh));
    if (c + 1 < nch) tma_prefetch_l2_3d(maps[which], 0, (c + 1) * C, static_cast<int>(bh));
    if (c + 1 < nch) tma_prefetch_l2_3d(maps[which], 64, (c + 1) * C, static_cast<int>(bh));
    ++issued[which];
  };
  if (tid == 0) {
    for (int b = 0; b < kNumBars; ++b) mbar_init(bar(b), 1);
    *flag = 0;
    fence_mbar_init();
    for (int b = 0; b < 4; ++b) tma_prefetch_desc(maps[b]);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  if (tid < 128) {
    pw[tid] = pow_int(L, tid);
    dpw[tid] = tid == 0 ? 0.f : static_cast<float>(tid) * pow_int(L, tid - 1);
    pwr[tid] = pow_int(L, C - 1 - tid);
    zt[tid] = 0.f;
    sv[tid] = 0.f;
  }
  if (tid == 0) {
    pw[C] = pow_int(L, C);
    dpw[C] = static_cast<float>(C) * pow_int(L, C - 1);
  }
  fill_masked_tables(L, tid, lo, dlo, nullptr);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lf = static_cast<uint32_t>((warp & 3) * 32) << 16;
  if (tid == 0 && c0 < c1)
    for (int b = 0; b < 4; ++b) load(b, c0);
  float geo = 0.f;   // sum_s lambda^(C-1-s) over a chunk
  for (int m = 0; m < C; ++m) geo += pwr[m];
  if (tid < 128) {
    float g = 0.f;
    for (int m = 0; m <= tid; ++m) g += pw[m];
    gs[tid] = g;
  }
  // thread 0 waits (bounded); every thread learns the verdict at the barrier
  auto poll = [&](int b, int parity) {
    if (tid == 0 && !*flag) {
      if (!mbar_wait(bar(b), static_cast<uint32_t>(parity) & 1u)) *flag = 1;
      else if (b <= kFullG) ++waited[b];
    }
  };
  auto meet = [&]() -> bool {
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    return *flag == 0;
  };
  int mph = 0;   // completed phases of the MMA barrier
  auto mma_done = [&]() { poll(kMma, mph); ++mph; };
  int mph2 = 0;  // completed phases of the second MMA barrier (a product an epilogue needs later)
  auto mma2_done = [&]() { poll(kMma2, mph2); ++mph2; };
  // Every thread waits for an MMA phase itself (no block barrier): a thread
  // whose wait runs out sets the flag and goes on to the next block barrier,
  // where all threads leave together.  A block barrier lies between any two
  // phases of each MMA barrier, so no thread is ever two phases behind.
  auto mma_wait_all = [&](int b, int &ph) {
    if (!*flag && !mbar_wait(bar(b), static_cast<uint32_t>(ph) & 1u)) *flag = 1;
    ++ph;
    tc_fence_after();
  };

  const uint64_t dQ = kdesc(sb + kOffQ), dK = kdesc(sb + kOffK), dKm = mdesc(sb + kOffK);
  const uint64_t dV = kdesc(sb + kOffV), dVm = mdesc(sb + kOffV);
  const uint64_t dSb = kdesc(sb + kOffSb), dSbm = mdesc(sb + kOffSb);
  float dl = 0.f;      // this thread's share of dlambda
  float zeta = 0.f;    // sum of the decay weights of the keys before the chunk
  if (half == 1) {
    // the state at token H0 C, from the state pass (this grid's prerequisite)
    grid_dependency_wait();
    const float *m = mid + bh * kMidFloats;
#pragma unroll 1
    for (int blk = hf; blk < hf + 1; ++blk) {
      uint32_t v[32];
      const float4 *src = reinterpret_cast<const float4 *>(m + i * D + blk * 32);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float4 x = src[e];
        v[4 * e] = __float_as_uint(x.x);
        v[4 * e + 1] = __float_as_uint(x.y);
        v[4 * e + 2] = __float_as_uint(x.z);
        v[4 * e + 3] = __float_as_uint(x.w);
      }
      tmem_st_32x32b_x32(tmem + kTmS + lf + blk * 32, v);
    }
    tmem_wait_st();
    if (tid < 128) {
      sv[i] = m[D * D + i];
      zt[i] = m[D * D + D + i];
    }
    zeta = m[D * D + 2 * D];
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }
  uint8_t *ap_row = sm + kOffAp + static_cast<uint32_t>(i) * 256u;   // At' row (its two halves)
  const int b0 = hf;   // this part's 32-column block
  const float lf_i = pw[i + 1];
  const float *mk = lo + 127 - i, *dmk = dlo + 127 - i;   // mk[s] = lambda^(i-s) (s <= i) or 0

  for (int c = c0; c < c1; ++c) {
    const int row0 = c * C, Cv = min(C, N - row0);
    const bool carried = c > c0 || half == 1, last = c == c1 - 1;
    // ---- the state before this chunk: bf16 operand, and lambda^C St kept for the update
    if (carried) state_to_operand<kParts>(tmem + kTmS + lf, sm + kOffSb, i, hf, pw[C]);
    poll(kFullQ, c - c0);
    if (!meet()) break;
    {
      float rqh = 0.f;
      X.put(kXQz, phi_row<kParts>(sm + kOffQ, i, hf, ident, zt, &rqh));   // phi(q_i) . zt, part
      X.put(kXRq, rqh);
    }
    poll(kFullK, c - c0);
    if (!meet()) break;
    const float rq = X.get(kXRq), qzt = X.get(kXQz);
    const float qz = qzt + o * rq * zeta;   // phi(q_i) . z
    elu_row<kParts>(sm + kOffK, i, hf, ident);
    fence_proxy_async_smem();
    if (!meet()) break;
    if (tid == 0) {
      mma_ss(tmem + kTmT1, dQ, false, dK, false, false);                 // Q Kt^T
      umma_commit(bar(kMma));
      if (carried) {
        mma_ss(tmem + kTmT2, dQ, false, dSbm, true, false);   // Q St, read after the next product
        umma_commit(bar(kMma2));
      }
    }
    mma_wait_all(kMma, mph);
    // ---- At = (Q Kt^T) o M into TMEM (bf16), At' = (Q Kt^T) o M' into shared memory
    {
      // this part's 32 columns in steps of 16 (x = the step's first column)
      float rsh = 0.f;
#pragma unroll 1
      for (int x = 32 * b0; x < 32 * b0 + 32; x += 16) {
        uint32_t v[16];
        tmem_ld_32x32b_x16(tmem + lf + kTmT1 + x, v);
        tmem_wait_ld();
        uint32_t pa[8], pp[8];
#pragma unroll
        for (int e = 0; e < 16; e += 2) {
          const int s0 = x + e, s1 = s0 + 1;
          const float p0 = __uint_as_float(v[e]), p1 = __uint_as_float(v[e + 1]);
          pa[e / 2] = pack_bf16(p0 * mk[s0], p1 * mk[s1]);
          rsh += blo(pa[e / 2]) + bhi(pa[e / 2]);
          pp[e / 2] = pack_bf16(p0 * dmk[s0], p1 * dmk[s1]);
        }
        tmem_st_32x32b_x8(tmem + lf + kTmA + x / 2, pa);
#pragma unroll
        for (int m = 0; m < 2; ++m)
          *reinterpret_cast<uint4 *>(ap_row + (((x / 8 + m) ^ (i & 15)) << 4)) =
              make_uint4(pp[4 * m], pp[4 * m + 1], pp[4 * m + 2], pp[4 * m + 3]);
      }
      X.put(kXRs, rsh);
    }
    tmem_wait_st();
    poll(kFullV, c - c0);
    if (!meet()) break;
    if (tid == 0) {
      mma_ts(tmem + kTmT1, tmem + kTmA, dVm, true, false);   // At V
      umma_commit(bar(kMma));
    }
    mma_done();
    if (carried) mma2_done();
    poll(kFullG, c - c0);
    if (!meet()) break;
    // ---- den, dnum (bf16 into TMEM) and dnum . num but for its o rq part
    const float den = lf_i * qz + o * rq * gs[i] + X.get(kXRs) + eps, inv = 1.f / den;
    {
      float gnh = 0.f, sdh = 0.f;   // dnum . (At V + carried part), dnum . s
#pragma unroll 1
      for (int x = 32 * b0; x < 32 * b0 + 32; x += 16) {
        uint32_t av[16], xv[16];
        tmem_ld_32x32b_x16(tmem + lf + kTmT1 + x, av);
        if (carried) tmem_ld_32x32b_x16(tmem + lf + kTmT2 + x, xv);
        tmem_wait_ld();
        uint32_t pk[8];
#pragma unroll
        for (int m = 0; m < 2; ++m) {
          const uint4 g4 = *reinterpret_cast<const uint4 *>(sm + kOffG + toff(i, x / 8 + m));
          const uint32_t g[4] = {g4.x, g4.y, g4.z, g4.w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int e = 8 * m + 2 * u, v0 = x + e;
            float n0 = __uint_as_float(av[e]), n1 = __uint_as_float(av[e + 1]);
            if (carried) {
              n0 += lf_i * (__uint_as_float(xv[e]) + o * rq * sv[v0]);
              n1 += lf_i * (__uint_as_float(xv[e + 1]) + o * rq * sv[v0 + 1]);
            }
            // dden from the bf16 dnum the MMAs use, so that dnum . v + dden (the
            // weight of every key) is exact up to the fp32 sums even where the
            // two terms nearly cancel
            pk[4 * m + u] = pack_bf16(blo(g[u]) * inv, bhi(g[u]) * inv);
            const float d0 = blo(pk[4 * m + u]), d1 = bhi(pk[4 * m + u]);
            gnh += d0 * n0 + d1 * n1;
            sdh += d0 * sv[v0] + d1 * sv[v0 + 1];
          }
        }
        tmem_st_32x32b_x8(tmem + lf + kTmW + x / 2, pk);
      }
      X.put(kXGn, gnh);
      X.put(kXSd, sdh);
    }
    tmem_wait_st();
    if (!meet()) break;
    if (tid == 0) {
      if (!last) load(3, c + 1);                                   // dy tile is free
      mma_ts(tmem + kTmT1, tmem + kTmW, dV, false, false);        // W = w V^T
      umma_commit(bar(kMma));
      if (carried) {
        mma_ts(tmem + kTmT2, tmem + kTmW, dSb, false, false);   // U = w St^T, read in the dq epilogue
        umma_commit(bar(kMma2));
      }
    }
    mma_wait_all(kMma, mph);
    const float gn = X.get(kXGn), sd = X.get(kXSd);
    // ---- dden = -dnum . num / den, the o rq part from the masked row sum of W
    {
      float gwh = 0.f;
#pragma unroll 1
      for (int blk = b0; blk < b0 + 1; ++blk) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tmem + lf + kTmT1 + blk * 32, v);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) gwh += __uint_as_float(v[e]) * mk[blk * 32 + e];
      }
      X.put(kXGw, gwh);
    }
    __syncthreads();
    const float dden = -(gn + o * rq * X.get(kXGw)) * inv;
    if (hf == 0 && i < Cv)
      *reinterpret_cast<float2 *>(stash + (bh * N + row0 + i) * stash_stride) =
          make_float2(den, dden);
    // ---- B = (W + dden) o M into TMEM, its fp32 row sum; dlambda, pairs inside the chunk
    {
      float rbh = 0.f;
#pragma unroll 1
      for (int x = 32 * b0; x < 32 * b0 + 32; x += 16) {
        uint32_t v[16];
        tmem_ld_32x32b_x16(tmem + lf + kTmT1 + x, v);
        tmem_wait_ld();
        uint32_t pb[8];
#pragma unroll
        for (int m = 0; m < 2; ++m) {
          const uint4 a4 = *reinterpret_cast<const uint4 *>(ap_row + (((x / 8 + m) ^ (i & 15)) << 4));
          const uint32_t ap[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int e = 8 * m + 2 * u;
            const int s0 = x + e, s1 = s0 + 1;
            const float w0 = __uint_as_float(v[e]) + dden, w1 = __uint_as_float(v[e + 1]) + dden;
            dl += (blo(ap[u]) + o * rq * dmk[s0]) * w0 + (bhi(ap[u]) + o * rq * dmk[s1]) * w1;
            const float bb0 = w0 * mk[s0], bb1 = w1 * mk[s1];
            rbh += bb0 + bb1;
            pb[4 * m + u] = pack_bf16(bb0, bb1);
          }
        }
        tmem_st_32x32b_x8(tmem + lf + kTmA + x / 2, pb);
      }
      X.put(kXRb, rbh);
    }
    tmem_wait_st();
    if (!meet()) break;
    if (tid == 0) {
      mma_ts(tmem + kTmT1, tmem + kTmA, dKm, true, false);   // B Kt
      umma_commit(bar(kMma));
    }
    mma_wait_all(kMma, mph);
    if (carried) mma_wait_all(kMma2, mph2);
    // ---- dq = (B Kt + o B1 + lambda^(t+1) (U + zt dden + o (s.w + zeta dden))) phi'(q);
    //      dlambda, keys before the chunk (the lambda^(t+1) factor's derivative)
    {
      float quh = 0.f;
      const float one = o * (X.get(kXRb) + (carried ? lf_i * (sd + zeta * dden) : 0.f));
      __nv_bfloat16 *dst = dq + (bh * N + row0 + i) * static_cast<long>(D);
#pragma unroll 1
      for (int x = 32 * b0; x < 32 * b0 + 32; x += 16) {
        uint32_t bk[16], uv[16];
        tmem_ld_32x32b_x16(tmem + lf + kTmT1 + x, bk);
        if (carried) tmem_ld_32x32b_x16(tmem + lf + kTmT2 + x, uv);
        tmem_wait_ld();
        uint32_t pk[8];
#pragma unroll
        for (int m = 0; m < 2; ++m) {
          const uint4 q4 = *reinterpret_cast<const uint4 *>(sm + kOffQ + toff(i, x / 8 + m));
          const uint32_t qw[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int e = 8 * m + 2 * u, k0 = x + e;
            const float u0 = carried ? __uint_as_float(uv[e]) : 0.f;
            const float u1 = carried ? __uint_as_float(uv[e + 1]) : 0.f;
            const float q0 = blo(qw[u]), q1 = bhi(qw[u]);
            quh += q0 * u0 + q1 * u1;
            float g0 = __uint_as_float(bk[e]) + one + lf_i * (u0 + dden * zt[k0]);
            float g1 = __uint_as_float(bk[e + 1]) + one + lf_i * (u1 + dden * zt[k0 + 1]);
            if (!ident) {
              g0 *= fminf(q0, 1.f);
              g1 *= fminf(q1, 1.f);
            }
            pk[4 * m + u] = pack_bf16(g0, g1);
          }
        }
        if (i < Cv)
#pragma unroll
          for (int m = 0; m < 2; ++m)
            reinterpret_cast<uint4 *>(dst + x)[m] =
                make_uint4(pk[4 * m], pk[4 * m + 1], pk[4 * m + 2], pk[4 * m + 3]);
      }
      if (carried)
        dl += dpw[i + 1] *
              (quh + (hf == 0 ? dden * qzt + o * rq * (sd + zeta * dden) : 0.f));
    }
    if (last) break;
    // ---- state update: key rows weighted lambda^(C-1-s): St += (Lk Kt)^T V, zt, s, zeta likewise
    scale_row<kParts>(sm + kOffK, sm + kOffK, i, hf, pwr[i]);
    fence_proxy_async_smem();
    if (!meet()) break;
    if (tid == 0) {
      mma_ss(tmem + kTmS, dKm, true, dVm, true, carried);
      umma_commit(bar(kMma));
      load(0, c + 1);   // the q tile is free
    }
    {
      // the At' tile is done with: its space holds the column-sum partials
      float zc = 0.f, sc = 0.f;
      col_sums<kNT>(sm + kOffK, nullptr, sm + kOffV, pwr, reinterpret_cast<float *>(sm + kOffAp),
                    zc, sc);
      if (tid < 128) {
        zt[i] = pw[C] * zt[i] + zc;
        sv[i] = pw[C] * sv[i] + sc;
      }
    }
    zeta = pw[C] * zeta + geo;
    mma_wait_all(kMma, mph);
    if (tid == 0) {
      load(1, c + 1);
      load(2, c + 1);
    }
  }
  // dlambda: pairs inside a chunk and the carried-state part of pairs across chunks
  if (dlam) {
    const float tot = block_sum(dl, red);
    if (tid == 0 && !*flag) atomicAdd(dlam + h, tot);
  }
  // leave with no copy and no MMA in flight
  if (tid == 0) {
    for (int b = 0; b < 4; ++b)
      for (int n = waited[b]; n < issued[b]; ++n) mbar_wait(bar(kFullQ + b), n & 1);
    umma_commit(bar(kFinal));
    mbar_wait(bar(kFinal), 0);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ============================================================== reverse state pass for split R
// Pass R can run as two CTAs per head: chunks [H1, nch) and [0, H1), each
// walked in reverse.  The second starts from the adjoint of every token at or
// after T = H1 C:
//   R = sum_{t>=T} lambda^(t-T+1) phi(q_t) w_t^T,   r = sum_{t>=T} lambda^(t-T+1) phi(q_t) dden_t
// which this pass sums over chunks [H1, nch) (q row t of chunk c weighted
// lambda^((c-H1) C) lambda^(t+1), no decay pass) and writes to `mid`: per
// head R [128][128] fp32, then r [128].
namespace pt {
constexpr uint32_t kOffQ0 = 0, kOffG0 = kTile, kStage = 2 * kTile, kOffMisc = 2 * kStage;
enum { kFullQ0 = 0, kFullG0, kFullQ1, kFullG1, kMma, kFinal, kNumBars };
constexpr uint32_t kMiscTmem = 64, kMiscFlag = 68, kMiscPw = 128;
constexpr uint32_t kMiscDd = kMiscPw + 132 * 4, kMiscScr = kMiscDd + 128 * 4;
constexpr int kNT = 512, kParts = 4;   // four warpgroups, a quarter of each row each
constexpr uint32_t kSmemBytes = kOffMisc + kMiscScr + 2 * (kNT / 32) * 128 * 4;
static_assert(kSmemBytes <= 232448, "exceeds the per-CTA shared memory of sm_100");
}  // namespace pt

__global__ void __launch_bounds__(pt::kNT, 1)
    bwd_tc_t_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_g,
                    const float *__restrict__ lam, const float *__restrict__ stash,
                    long stash_stride, float *__restrict__ mid, int H, int N, int H1, bool ident) {
  using namespace pt;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *sm = smem_raw;
  const uint32_t sb = smem_u32(sm);
  const int tid = threadIdx.x, warp = tid >> 5;
  if (sb & 1023u) {
    if (tid == 0) atomicOr(&g_status, kStatusWaitTimeout);
    return;
  }
  // pass R (launched next as this pass's programmatic dependent) starts its
  // later halves at once; its earlier halves wait for this grid
  grid_launch_dependents();
  const long bh = blockIdx.x;
  const int h = static_cast<int>(bh % H);
  const float L = lam ? lam[h] : 1.f;
  const int nch = (N + C - 1) / C, n = nch - H1;   // chunks H1 .. nch-1
  uint8_t *misc = sm + kOffMisc;
  auto bar = [&](int i) { return sb + kOffMisc + 8u * static_cast<uint32_t>(i); };
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(misc + kMiscTmem);
  volatile int *flag = reinterpret_cast<volatile int *>(misc + kMiscFlag);
  float *pw = reinterpret_cast<float *>(misc + kMiscPw);   // lambda^m, m = 0..C
  float *dd = reinterpret_cast<float *>(misc + kMiscDd);   // dden of the chunk's tokens
  float *scr = reinterpret_cast<float *>(misc + kMiscScr);
  const int hf = tid >> 7, i = tid & 127;
  int issued[4] = {0, 0, 0, 0}, waited[4] = {0, 0, 0, 0};
  auto load = [&](int j) {   // j-th chunk of the walk: chunk H1 + j
    const int st = j & 1, c = H1 + j;
    for (int which = 0; which < 2; ++which) {
      const CUtensorMap *map = which ? &tm_g : &tm_q;
      const int b = 2 * st + which;
      const uint32_t dst = sb + st * kStage + (which ? kOffG0 : kOffQ0);
      mbar_arrive_expect_tx(bar(b), kTile);
      tma_load_3d(dst, map, bar(b), 0, c * C, static_cast<int>(bh));
      tma_load_3d(dst + kPanel, map, bar(b), 64, c * C, static_cast<int>(bh));
      if (j + 2 < n) tma_prefetch_l2_3d(map, 0, (c + 2) * C, static_cast<int>(bh));
      if (j + 2 < n) tma_prefetch_l2_3d(map, 64, (c + 2) * C, static_cast<int>(bh));
      ++issued[b];
    }
  };
  if (tid == 0) {
    for (int b = 0; b < kNumBars; ++b) mbar_init(bar(b), 1);
    *flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_g);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), 128);
    tmem_relinquish();
  }
  if (tid < 128) pw[tid] = pow_int(L, tid);
  if (tid == 0) pw[C] = pow_int(L, C);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lf = static_cast<uint32_t>((warp & 3) * 32) << 16;
  if (tid == 0)
    for (int j = 0; j < min(n, 2); ++j) load(j);
  auto poll = [&](int b, int parity) {
    if (tid == 0 && !*flag) {
      if (!mbar_wait(bar(b), static_cast<uint32_t>(parity) & 1u)) *flag = 1;
      else if (b <= kFullG1) ++waited[b];
    }
  };
  auto meet = [&]() -> bool {
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    return *flag == 0;
  };
  int mph = 0;
  // every thread waits for the MMA phase itself (see pass F)
  auto mma_wait_all = [&](int b, int &ph) {
    if (!*flag && !mbar_wait(bar(b), static_cast<uint32_t>(ph) & 1u)) *flag = 1;
    ++ph;
    tc_fence_after();
  };
  float r_acc = 0.f;   // thread i < 128: column i of r

  for (int j = 0; j < n; ++j) {
    const int st = j & 1, c = H1 + j, row0 = c * C, Cv = min(C, N - row0);
    uint8_t *tq = sm + st * kStage + kOffQ0, *tg = sm + st * kStage + kOffG0;
    float den = 1.f, dden = 0.f;   // tokens past the end: no gradient
    if (i < Cv) {
      const float2 sv = *reinterpret_cast<const float2 *>(stash + (bh * N + row0 + i) * stash_stride);
      den = sv.x;
      dden = sv.y;
    }
    if (hf == 0) dd[i] = dden;
    poll(2 * st, j >> 1);
    poll(2 * st + 1, j >> 1);
    if (!meet()) break;
    phi_row<kParts>(tq, i, hf, ident, nullptr);
    scale_row<kParts>(tq, tq, i, hf, pow_int(L, j * C) * pw[i + 1]);
    dnum_row<kParts>(tg, i, hf, 1.f / den);
    fence_proxy_async_smem();
    if (!meet()) break;
    if (tid == 0) {
      mma_ss(tmem, mdesc(smem_u32(tq)), true, mdesc(smem_u32(tg)), true, j > 0);   // R += (Lq Q)^T w
      umma_commit(bar(kMma));
    }
    {
      float rc = 0.f, unused = 0.f;
      col_sums<kNT>(tq, dd, nullptr, nullptr, scr, rc, unused);
      if (tid < 128) r_acc += rc;
    }
    mma_wait_all(kMma, mph);
    if (tid == 0 && j + 2 < n) load(j + 2);   // this stage is free
  }
  if (!*flag && n > 0) {
    float *m = mid + bh * kMidFloats;
#pragma unroll 1
    for (int blk = hf; blk < hf + 1; ++blk) {
      uint32_t v[32];
      tmem_ld_32x32b_x32(tmem + lf + blk * 32, v);
      tmem_wait_ld();
      float4 *dst = reinterpret_cast<float4 *>(m + i * D + blk * 32);
#pragma unroll
      for (int e = 0; e < 8; ++e)
        dst[e] = make_float4(__uint_as_float(v[4 * e]), __uint_as_float(v[4 * e + 1]),
                             __uint_as_float(v[4 * e + 2]), __uint_as_float(v[4 * e + 3]));
    }
    if (tid < 128) m[D * D + i] = r_acc;
  }
  if (tid == 0) {
    for (int b = 0; b < 4; ++b)
      for (int k = waited[b]; k < issued[b]; ++k) mbar_wait(bar(b), k & 1);
    umma_commit(bar(kFinal));
    mbar_wait(bar(kFinal), 0);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// ============================================================== pass R
namespace pr {
constexpr uint32_t kOffQ = 0, kOffK = kTile, kOffKd = 2 * kTile, kOffV = 3 * kTile,
                   kOffVd = 4 * kTile, kOffG = 5 * kTile, kOffRb = 6 * kTile, kOffMisc = 7 * kTile;
enum { kFullQ = 0, kFullK, kFullV, kFullG, kMma, kMma2, kFinal, kNumBars };
constexpr uint32_t kMiscTmem = 64, kMiscFlag = 68, kMiscUp = 128;
constexpr uint32_t kMiscDden = kMiscUp + 256 * 4, kMiscR = kMiscDden + 128 * 4;
constexpr uint32_t kSmemBytes = kOffMisc + kMiscR + 128 * 4;
static_assert(kSmemBytes <= 232448, "exceeds the per-CTA shared memory of sm_100");
constexpr uint32_t kTmR = 0, kTmT1 = 128, kTmT2 = 256, kTmAt = 384, kTmBt = 448;
// four warpgroups: thread (h, r) owns the 32 columns [32h, 32h + 32) of row r
// (the reverse pass has no row sums to join, so more warps only add latency
// hiding)
constexpr int kNT = 512, kParts = 4;
}  // namespace pr

__global__ void __launch_bounds__(pr::kNT, 1)
    bwd_tc_r_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
                    const float *__restrict__ lam, const float *stash, long stash_stride,
                    __nv_bfloat16 *__restrict__ dk, __nv_bfloat16 *__restrict__ dv,
                    const float *__restrict__ rmid, int H1, int H, int N, bool ident) {
  using namespace pr;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *sm = smem_raw;
  const uint32_t sb = smem_u32(sm);
  const int tid = threadIdx.x, warp = tid >> 5;
  if (sb & 1023u) {
    if (tid == 0) atomicOr(&g_status, kStatusWaitTimeout);
    return;
  }
  // H1 > 0: two CTAs per head, chunks [H1, nch) and [0, H1), each walked in
  // reverse; the second starts from the adjoint the reverse state pass leaves in `rmid`
  const int G = H1 > 0 ? 2 : 1;
  const long BH = gridDim.x / G;
  const int half = static_cast<int>(blockIdx.x / BH);
  const long bh = blockIdx.x % BH;
  const int h = static_cast<int>(bh % H);
  const float L = lam ? lam[h] : 1.f;
  const int nch = (N + C - 1) / C;
  const int c_lo = half ? 0 : H1, c_hi = half ? H1 : nch;   // chunks [c_lo, c_hi)
  uint8_t *misc = sm + kOffMisc;
  auto bar = [&](int i) { return sb + kOffMisc + 8u * static_cast<uint32_t>(i); };
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(misc + kMiscTmem);
  volatile int *flag = reinterpret_cast<volatile int *>(misc + kMiscFlag);
  // up[127 - t + s] = lambda^(s-t) for s >= t, else 0; up[127 + m] = lambda^m for m = 0..128
  float *up = reinterpret_cast<float *>(misc + kMiscUp);
  const float *pw = up + 127;
  float *sdd = reinterpret_cast<float *>(misc + kMiscDden);   // dden of the chunk's tokens
  float *rv = reinterpret_cast<float *>(misc + kMiscR);       // r, the normaliser's adjoint
  const int hf = tid >> 7, i = tid & 127;
  const CUtensorMap *maps[4] = {&tm_q, &tm_k, &tm_v, &tm_g};
  int issued[4] = {0, 0, 0, 0}, waited[4] = {0, 0, 0, 0};
  // Tile roles alternate between chunks: the q and dy tiles of the next chunk
  // are loaded into this chunk's weighted k and v buffers once the dv and dk
  // products have read them, and the next chunk weights k and v into this
  // chunk's q and dy buffers.  With parity 0 the roles sit in the buffers
  // named for them; with parity 1 q and weighted k trade buffers, and so do
  // dy and weighted v.
  auto off_q = [](int p) { return p ? kOffKd : kOffQ; };
  auto off_g = [](int p) { return p ? kOffVd : kOffG; };
  auto off_kd = [](int p) { return p ? kOffQ : kOffKd; };
  auto off_vd = [](int p) { return p ? kOffG : kOffVd; };
  auto load = [&](int which, int c, uint32_t off) {
    const uint32_t b = bar(kFullQ + which);
    mbar_arrive_expect_tx(b, kTile);
    tma_load_3d(sb + off, maps[which], b, 0, c * C, static_cast<int>(bh));
    tma_load_3d(sb + off + kPanel, maps[which], b, 64, c * C, static_cast<int>(bh));
    if (c > 0) tma_prefetch_l2_3d(maps[which], 0, (c - 1) * C, static_cast<int>(bh));
    if (c > 0) tma_prefetch_l2_3d(maps[which], 64, (c - 1) * C, static_cast<int>(bh));
    ++issued[which];
  };
  if (tid == 0) {
    for (int b = 0; b < kNumBars; ++b) mbar_init(bar(b), 1);
    *flag = 0;
    fence_mbar_init();
    for (int b = 0; b < 4; ++b) tma_prefetch_desc(maps[b]);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  fill_masked_tables(L, tid, nullptr, nullptr, up);
  if (tid < 128) rv[tid] = 0.f;
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lf = static_cast<uint32_t>((warp & 3) * 32) << 16;
  if (tid == 0 && c_lo < c_hi) {
    load(0, c_hi - 1, off_q(0));
    load(1, c_hi - 1, kOffK);
    load(2, c_hi - 1, kOffV);
    load(3, c_hi - 1, off_g(0));
  }
  auto poll = [&](int b, int parity) {
    if (tid == 0 && !*flag) {
      if (!mbar_wait(bar(b), static_cast<uint32_t>(parity) & 1u)) *flag = 1;
      else if (b <= kFullG) ++waited[b];
    }
  };
  auto meet = [&]() -> bool {
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    return *flag == 0;
  };
  int mph = 0;   // completed phases of the MMA barrier
  int mph2 = 0;  // completed phases of the second MMA barrier (a product an epilogue needs later)
  // Every thread waits for an MMA phase itself (no block barrier): a thread
  // whose wait runs out sets the flag and goes on to the next block barrier,
  // where all threads leave together.  A block barrier lies between any two
  // phases of each MMA barrier, so no thread is ever two phases behind.
  auto mma_wait_all = [&](int b, int &ph) {
    if (!*flag && !mbar_wait(bar(b), static_cast<uint32_t>(ph) & 1u)) *flag = 1;
    ++ph;
    tc_fence_after();
  };

  const uint64_t dK = kdesc(sb + kOffK), dV = kdesc(sb + kOffV);
  const uint64_t dRb = kdesc(sb + kOffRb), dRbm = mdesc(sb + kOffRb);
  const int b0 = hf;   // this part's 32-column block
  const float *mk = up + 127 - i;   // mk[s] = lambda^(s-i) for s >= i, else 0
  // den, dden of this thread's token in the chunk being processed (tokens past
  // the end: no gradient); the next chunk's pair is loaded a chunk ahead
  float2 st = make_float2(1.f, 0.f);
  if (c_lo < c_hi && i < N - (c_hi - 1) * C)
    st = *reinterpret_cast<const float2 *>(stash + (bh * N + (c_hi - 1) * C + i) * stash_stride);
  if (half == 1) {
    // the adjoint of the tokens from H1 C on, from the reverse state pass
    // (this grid's prerequisite)
    grid_dependency_wait();
    const float *m = rmid + bh * kMidFloats;
#pragma unroll 1
    for (int blk = hf; blk < hf + 1; ++blk) {
      uint32_t v[32];
      const float4 *src = reinterpret_cast<const float4 *>(m + i * D + blk * 32);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float4 x = src[e];
        v[4 * e] = __float_as_uint(x.x);
        v[4 * e + 1] = __float_as_uint(x.y);
        v[4 * e + 2] = __float_as_uint(x.z);
        v[4 * e + 3] = __float_as_uint(x.w);
      }
      tmem_st_32x32b_x32(tmem + kTmR + lf + blk * 32, v);
    }
    tmem_wait_st();
    if (tid < 128) rv[i] = m[D * D + i];
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }

  for (int cc = 0; cc < c_hi - c_lo; ++cc) {
    const int c = c_hi - 1 - cc, row0 = c * C, Cv = min(C, N - row0);
    const bool carried = cc > 0 || half == 1;   // later tokens exist: R, r nonzero
    const int par = cc & 1;
    const uint32_t oQ = off_q(par), oG = off_g(par), oKd = off_kd(par), oVd = off_vd(par);
    const uint64_t dQ = kdesc(sb + oQ), dQm = mdesc(sb + oQ), dG = kdesc(sb + oG),
                   dGm = mdesc(sb + oG), dKd = kdesc(sb + oKd), dVd = kdesc(sb + oVd);
    const float den = st.x, dden = st.y;
    if (hf == 0) sdd[i] = dden;
    if (carried) state_to_operand<kParts>(tmem + kTmR + lf, sm + kOffRb, i, hf, pw[C]);
    poll(kFullQ, cc);
    poll(kFullK, cc);
    poll(kFullV, cc);
    poll(kFullG, cc);
    if (!meet()) break;
    phi_row<kParts>(sm + oQ, i, hf, ident, nullptr);
    phi_row<kParts>(sm + kOffK, i, hf, ident, nullptr);
    if (carried) {
      scale_row<kParts>(sm + oKd, sm + kOffK, i, hf, pw[C - 1 - i]);
      scale_row<kParts>(sm + oVd, sm + kOffV, i, hf, pw[C - 1 - i]);
    }
    dnum_row<kParts>(sm + oG, i, hf, 1.f / den);   // w = dnum in place of dy
    fence_proxy_async_smem();
    if (!meet()) break;
    if (tid == 0) {
      mma_ss(tmem + kTmT1, dK, false, dQ, false, false);   // P^T = K Q^T
      umma_commit(bar(kMma));
      mma_ss(tmem + kTmT2, dV, false, dG, false, false);   // W^T = V w^T
      umma_commit(bar(kMma2));
    }
    // the next chunk's den, dden, while the products run
    if (c > c_lo)
      st = *reinterpret_cast<const float2 *>(stash + (bh * N + row0 - C + i) * stash_stride);
    mma_wait_all(kMma, mph);
    // ---- A^T and B^T rows (key i, queries s >= i) into TMEM
#pragma unroll 1
    for (int blk = b0; blk < b0 + 1; ++blk) {
      uint32_t pv[32];
      tmem_ld_32x32b_x32(tmem + lf + kTmT1 + blk * 32, pv);
      tmem_wait_ld();
      uint32_t pa[16];
#pragma unroll
      for (int e = 0; e < 32; e += 2)
        pa[e / 2] = pack_bf16(__uint_as_float(pv[e]) * mk[blk * 32 + e],
                              __uint_as_float(pv[e + 1]) * mk[blk * 32 + e + 1]);
      tmem_st_32x32b_x16(tmem + lf + kTmAt + blk * 16, pa);
    }
    mma_wait_all(kMma2, mph2);
    if (tid == 0 && c > c_lo) load(2, c - 1, kOffV);   // v has been read (its weighted copy is made)
#pragma unroll 1
    for (int blk = b0; blk < b0 + 1; ++blk) {
      uint32_t wv[32];
      tmem_ld_32x32b_x32(tmem + lf + kTmT2 + blk * 32, wv);
      tmem_wait_ld();
      uint32_t pb[16];
#pragma unroll
      for (int e = 0; e < 32; e += 2) {
        const int s0 = blk * 32 + e, s1 = s0 + 1;
        pb[e / 2] = pack_bf16((__uint_as_float(wv[e]) + sdd[s0]) * mk[s0],
                              (__uint_as_float(wv[e + 1]) + sdd[s1]) * mk[s1]);
      }
      tmem_st_32x32b_x16(tmem + lf + kTmBt + blk * 16, pb);
    }
    tmem_wait_st();
    if (!meet()) break;
    if (tid == 0) {
      mma_ts(tmem + kTmT1, tmem + kTmAt, dGm, true, false);                 // A^T w
      if (carried) mma_ss(tmem + kTmT1, dKd, false, dRbm, true, true);     // + Lk K R
      umma_commit(bar(kMma));
      mma_ts(tmem + kTmT2, tmem + kTmBt, dQm, true, false);                 // B^T Q
      if (carried) mma_ss(tmem + kTmT2, dVd, false, dRb, false, true);     // + Lk V R^T
      umma_commit(bar(kMma2));
    }
    mma_wait_all(kMma, mph);
    // ---- dv (while the dk product runs), then dk = (dphi(k) + Lk r) phi'(k)
    {
      __nv_bfloat16 *vd = dv + (bh * N + row0 + i) * static_cast<long>(D);
#pragma unroll 1
      for (int blk = b0; blk < b0 + 1; ++blk) {
        uint32_t a[32];
        tmem_ld_32x32b_x32(tmem + lf + kTmT1 + blk * 32, a);
        tmem_wait_ld();
        uint32_t pv[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2)
          pv[e / 2] = pack_bf16(__uint_as_float(a[e]), __uint_as_float(a[e + 1]));
        if (i < Cv)
#pragma unroll
          for (int m = 0; m < 4; ++m)
            reinterpret_cast<uint4 *>(vd + blk * 32)[m] =
                make_uint4(pv[4 * m], pv[4 * m + 1], pv[4 * m + 2], pv[4 * m + 3]);
      }
    }
    mma_wait_all(kMma2, mph2);
    if (tid == 0 && c > c_lo) {
      // the weighted k and v tiles have been read: the next chunk's q and dy go there
      load(0, c - 1, off_q(par ^ 1));
      load(3, c - 1, off_g(par ^ 1));
    }
    {
      const float kf = carried ? pw[C - 1 - i] : 0.f;
      __nv_bfloat16 *kd = dk + (bh * N + row0 + i) * static_cast<long>(D);
#pragma unroll 1
      for (int blk = b0; blk < b0 + 1; ++blk) {
        uint32_t b[32];
        tmem_ld_32x32b_x32(tmem + lf + kTmT2 + blk * 32, b);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const uint4 k4 = *reinterpret_cast<const uint4 *>(sm + kOffK + toff(i, blk * 4 + m));
          const uint32_t kw[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int e = 8 * m + 2 * u, k0 = blk * 32 + e;
            float g0 = __uint_as_float(b[e]) + kf * rv[k0];
            float g1 = __uint_as_float(b[e + 1]) + kf * rv[k0 + 1];
            if (!ident) {
              g0 *= fminf(blo(kw[u]), 1.f);
              g1 *= fminf(bhi(kw[u]), 1.f);
            }
            pk[4 * m + u] = pack_bf16(g0, g1);
          }
        }
        if (i < Cv)
#pragma unroll
          for (int m = 0; m < 4; ++m)
            reinterpret_cast<uint4 *>(kd + blk * 32)[m] =
                make_uint4(pk[4 * m], pk[4 * m + 1], pk[4 * m + 2], pk[4 * m + 3]);
      }
    }
    if (c == c_lo) break;   // the adjoint before the range is not needed here
    // ---- R += (Lq Q)^T w, r likewise: q rows weighted lambda^(t+1)
    scale_row<kParts>(sm + oQ, sm + oQ, i, hf, pw[i + 1]);
    fence_proxy_async_smem();
    if (!meet()) break;
    if (tid == 0) {
      mma_ss(tmem + kTmR, dQm, true, dGm, true, carried);
      umma_commit(bar(kMma));
      load(1, c - 1, kOffK);   // k has been read
    }
    {
      // the bf16 R operand is done with until the next chunk: its space holds
      // the column-sum partials
      float rc = 0.f, unused = 0.f;
      col_sums<kNT>(sm + oQ, sdd, nullptr, nullptr, reinterpret_cast<float *>(sm + kOffRb), rc,
                    unused);
      if (tid < 128) rv[i] = pw[C] * rv[i] + rc;
    }
    mma_wait_all(kMma, mph);
  }
  if (tid == 0) {
    for (int b = 0; b < 4; ++b)
      for (int n = waited[b]; n < issued[b]; ++n) mbar_wait(bar(kFullQ + b), n & 1);
    umma_commit(bar(kFinal));
    mbar_wait(bar(kFinal), 0);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ============================================================== pass L
// dlambda's part from the derivative state S' = dS/dlambda (keys before the
// chunk), in the elu form of pass F: S' = St' + o 1 s'^T, z' = zt' + o zeta' 1,
//   <S', Ms> = <St', Ms> + o s' . (1^T Ms),   1^T Ms = sum_t lambda^(t+1) rq_t w_t
//   sum_t dden_t lambda^(t+1) Q_t . z' = sum_t dden_t lambda^(t+1) (Q_t . zt' + o rq_t zeta')
// and every part of (St, s, zt, zeta) and of its derivative steps per chunk as
//   X' <- lambda^C X' + C lambda^(C-1) X + (chunk term with (C-1-s) lambda^(C-2-s))
//   X  <- lambda^C X  + (chunk term with lambda^(C-1-s)).
namespace pl {
constexpr uint32_t kOffQ = 0, kOffK = kTile, kOffKp = 2 * kTile, kOffV = 3 * kTile,
                   kOffG = 4 * kTile, kOffMisc = 5 * kTile;
enum { kFullQ = 0, kFullK, kFullV, kFullG, kMma, kMma2, kFinal, kNumBars };
constexpr uint32_t kMiscTmem = 64, kMiscFlag = 68, kMiscPw = 128;
constexpr uint32_t kMiscDpw = kMiscPw + 132 * 4, kMiscPwr = kMiscDpw + 132 * 4;
constexpr uint32_t kMiscDpwr = kMiscPwr + 128 * 4, kMiscZ = kMiscDpwr + 128 * 4;
constexpr uint32_t kMiscZp = kMiscZ + 128 * 4, kMiscS = kMiscZp + 128 * 4;
constexpr uint32_t kMiscSp = kMiscS + 128 * 4, kMiscWq = kMiscSp + 128 * 4;
// four warpgroups: thread (h, r) owns the 32 columns [32h, 32h + 32) of row r
constexpr int kNT = 512, kParts = 4;
constexpr uint32_t kMiscRed = kMiscWq + 128 * 4, kMiscX = kMiscRed + 64;
enum { kXQz = 0, kXRq, kNumX };
constexpr uint32_t kMiscScr = kMiscX + kNumX * kParts * 128 * 4;   // column-sum partials
constexpr uint32_t kSmemBytes = kOffMisc + kMiscScr + 2 * (kNT / 32) * 128 * 4;
static_assert(kSmemBytes <= 232448, "exceeds the per-CTA shared memory of sm_100");
constexpr uint32_t kTmS = 0, kTmSp = 128, kTmM = 256;
}  // namespace pl

__global__ void __launch_bounds__(pl::kNT, 1)
    bwd_tc_l_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
                    const float *__restrict__ lam, const float *__restrict__ stash,
                    long stash_stride, float *__restrict__ dlam, int H, int N, bool ident) {
  using namespace pl;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *sm = smem_raw;
  const uint32_t sb = smem_u32(sm);
  const int tid = threadIdx.x, warp = tid >> 5;
  if (sb & 1023u) {
    if (tid == 0) atomicOr(&g_status, kStatusWaitTimeout);
    return;
  }
  const long bh = blockIdx.x;
  const int h = static_cast<int>(bh % H);
  const float L = lam ? lam[h] : 1.f;
  const float o = ident ? 0.f : 1.f;
  const int nch = (N + C - 1) / C;
  uint8_t *misc = sm + kOffMisc;
  auto bar = [&](int i) { return sb + kOffMisc + 8u * static_cast<uint32_t>(i); };
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(misc + kMiscTmem);
  volatile int *flag = reinterpret_cast<volatile int *>(misc + kMiscFlag);
  float *pw = reinterpret_cast<float *>(misc + kMiscPw);
  float *dpw = reinterpret_cast<float *>(misc + kMiscDpw);
  float *pwr = reinterpret_cast<float *>(misc + kMiscPwr);     // lambda^(C-1-s)
  float *dpwr = reinterpret_cast<float *>(misc + kMiscDpwr);   // (C-1-s) lambda^(C-2-s)
  float *zt = reinterpret_cast<float *>(misc + kMiscZ);
  float *ztp = reinterpret_cast<float *>(misc + kMiscZp);
  float *sv = reinterpret_cast<float *>(misc + kMiscS);
  float *svp = reinterpret_cast<float *>(misc + kMiscSp);
  float *wq = reinterpret_cast<float *>(misc + kMiscWq);       // lambda^(t+1) rq_t
  float *red = reinterpret_cast<float *>(misc + kMiscRed);
  float *scr = reinterpret_cast<float *>(misc + kMiscScr);
  const int hf = tid >> 7, i = tid & 127;
  const Halves X{reinterpret_cast<float *>(misc + kMiscX), hf, i, kParts};
  const CUtensorMap *maps[4] = {&tm_q, &tm_k, &tm_v, &tm_g};
  const uint32_t offs[4] = {kOffQ, kOffK, kOffV, kOffG};
  int issued[4] = {0, 0, 0, 0}, waited[4] = {0, 0, 0, 0};
  auto load = [&](int which, int c) {
    const uint32_t b = bar(kFullQ + which);
    mbar_arrive_expect_tx(b, kTile);
    tma_load_3d(sb + offs[which], maps[which], b, 0, c * C, static_cast<int>(bh));
    tma_load_3d(sb + offs[which] + kPanel, maps[which], b, 64, c * C, static_cast<int>(bh));
    if (c + 1 < nch) tma_prefetch_l2_3d(maps[which], 0, (c + 1) * C, static_cast<int>(bh));
    if (c + 1 < nch) tma_prefetch_l2_3d(maps[which], 64, (c + 1) * C, static_cast<int>(bh));
    ++issued[which];
  };
  if (tid == 0) {
    for (int b = 0; b < kNumBars; ++b) mbar_init(bar(b), 1);
    *flag = 0;
    fence_mbar_init();
    for (int b = 0; b < 4; ++b) tma_prefetch_desc(maps[b]);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  if (tid < 128) {
    pw[tid] = pow_int(L, tid);
    dpw[tid] = tid == 0 ? 0.f : static_cast<float>(tid) * pow_int(L, tid - 1);
    pwr[tid] = pow_int(L, C - 1 - tid);
    dpwr[tid] = tid == C - 1 ? 0.f : static_cast<float>(C - 1 - tid) * pow_int(L, C - 2 - tid);
    zt[tid] = 0.f;
    ztp[tid] = 0.f;
    sv[tid] = 0.f;
    svp[tid] = 0.f;
  }
  if (tid == 0) {
    pw[C] = pow_int(L, C);
    dpw[C] = static_cast<float>(C) * pow_int(L, C - 1);
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lf = static_cast<uint32_t>((warp & 3) * 32) << 16;
  if (tid == 0 && nch > 0)
    for (int b = 0; b < 4; ++b) load(b, 0);
  // the reverse pass (launched after this one as its programmatic dependent,
  // when the stash is not in dk) reads nothing this pass writes: let it start
  grid_launch_dependents();
  auto poll = [&](int b, int parity) {
    if (tid == 0 && !*flag) {
      if (!mbar_wait(bar(b), static_cast<uint32_t>(parity) & 1u)) *flag = 1;
      else if (b <= kFullG) ++waited[b];
    }
  };
  auto meet = [&]() -> bool {
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    return *flag == 0;
  };
  int mph = 0;   // completed phases of the MMA barrier
  // Every thread waits for an MMA phase itself (no block barrier): a thread
  // whose wait runs out sets the flag and goes on to the next block barrier,
  // where all threads leave together.  A block barrier lies between any two
  // phases of each MMA barrier, so no thread is ever two phases behind.
  auto mma_wait_all = [&](int b, int &ph) {
    if (!*flag && !mbar_wait(bar(b), static_cast<uint32_t>(ph) & 1u)) *flag = 1;
    ++ph;
    tc_fence_after();
  };

  const uint64_t dQm = mdesc(sb + kOffQ), dKm = mdesc(sb + kOffK), dKpm = mdesc(sb + kOffKp);
  const uint64_t dVm = mdesc(sb + kOffV), dGm = mdesc(sb + kOffG);
  const int b0 = hf;   // this part's 32-column block
  float dl = 0.f;
  float zeta = 0.f, zetap = 0.f;
  float geo = 0.f, dgeo = 0.f;
  for (int m = 0; m < C; ++m) {
    geo += pwr[m];
    dgeo += dpwr[m];
  }

  // den, dden of this thread's token in the chunk (past the end: no
  // gradient); the next chunk's pair is loaded a chunk ahead
  float2 st = make_float2(1.f, 0.f);
  if (nch > 0 && i < min(C, N))
    st = *reinterpret_cast<const float2 *>(stash + (bh * N + i) * stash_stride);

  for (int c = 0; c < nch; ++c) {
    const int row0 = c * C;
    const bool carried = c > 0, last = c == nch - 1;
    const float den = st.x, dden = st.y;
    poll(kFullQ, c);
    poll(kFullK, c);
    poll(kFullV, c);
    poll(kFullG, c);
    if (!meet()) break;
    // q rows weighted lambda^(t+1); the half sums of phi(q) . zt' and of phi(q)
    {
      float rqh = 0.f;
      X.put(kXQz, phi_row<kParts>(sm + kOffQ, i, hf, ident, ztp, &rqh));
      X.put(kXRq, rqh);
    }
    scale_row<kParts>(sm + kOffQ, sm + kOffQ, i, hf, pw[i + 1]);
    dnum_row<kParts>(sm + kOffG, i, hf, 1.f / den);
    if (!last) {
      // key rows as elu(k), weighted lambda^(C-1-s) (state) and (C-1-s) lambda^(C-2-s) (derivative)
      elu_row<kParts>(sm + kOffK, i, hf, ident);
      scale_row<kParts>(sm + kOffKp, sm + kOffK, i, hf, dpwr[i]);
      scale_row<kParts>(sm + kOffK, sm + kOffK, i, hf, pwr[i]);
    }
    fence_proxy_async_smem();
    if (!meet()) break;
    if (tid == 0) {
      mma_ss(tmem + kTmM, dQm, true, dGm, true, false);   // Ms = (Lq Q)^T w
      umma_commit(bar(kMma));
    }
    st = make_float2(1.f, 0.f);   // the next chunk's den, dden
    if (!last && i < N - row0 - C)
      st = *reinterpret_cast<const float2 *>(stash + (bh * N + row0 + C + i) * stash_stride);
    {
      // the z' part of dlambda (once per row), and lambda^(t+1) rq_t for 1^T Ms
      const float rq = X.get(kXRq);
      if (hf == 0) {
        dl += dden * pw[i + 1] * (X.get(kXQz) + o * rq * zetap);
        wq[i] = pw[i + 1] * rq;
      }
    }
    __syncthreads();   // wq is complete
    {
      // o s' . (1^T Ms) on this thread's d_v column (s' of the chunk start)
      float cs = 0.f, unused = 0.f;
      col_sums<kNT>(sm + kOffG, wq, nullptr, nullptr, scr, cs, unused);
      if (tid < 128) dl += o * svp[i] * cs;
    }
    mma_wait_all(kMma, mph);
    if (tid == 0 && !last) {
      load(0, c + 1);
      load(3, c + 1);
    }
    // <St', Ms> on this thread's d_k row; then St' <- lambda^C St' + C lambda^(C-1) St, St <- lambda^C St
    if (carried) {
      // this part's 32 columns in two steps of 16 (three values live per column)
#pragma unroll 1
      for (int col = 32 * b0; col < 32 * b0 + 32; col += 16) {
        uint32_t sp[16], mv[16], sq[16];
        tmem_ld_32x32b_x16(tmem + lf + kTmSp + col, sp);
        tmem_ld_32x32b_x16(tmem + lf + kTmM + col, mv);
        tmem_ld_32x32b_x16(tmem + lf + kTmS + col, sq);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float s1 = __uint_as_float(sp[e]), s0 = __uint_as_float(sq[e]);
          dl += s1 * __uint_as_float(mv[e]);
          sp[e] = __float_as_uint(pw[C] * s1 + dpw[C] * s0);
          sq[e] = __float_as_uint(pw[C] * s0);
        }
        if (!last) {
          tmem_st_32x32b_x16(tmem + lf + kTmSp + col, sp);
          tmem_st_32x32b_x16(tmem + lf + kTmS + col, sq);
        }
      }
      tmem_wait_st();
    }
    if (last) break;
    // the vector parts of the state and of its derivative: half sums over the chunk's rows
    if (!meet()) break;
    if (tid == 0) {
      mma_ss(tmem + kTmS, dKm, true, dVm, true, carried);
      mma_ss(tmem + kTmSp, dKpm, true, dVm, true, carried);
      umma_commit(bar(kMma));
    }
    {
      float zpc = 0.f, zc = 0.f, spc = 0.f, sc = 0.f;
      col_sums<kNT>(sm + kOffKp, nullptr, sm + kOffK, nullptr, scr, zpc, zc);
      col_sums<kNT>(sm + kOffV, dpwr, sm + kOffV, pwr, scr, spc, sc);
      if (tid < 128) {
        ztp[i] = pw[C] * ztp[i] + dpw[C] * zt[i] + zpc;
        zt[i] = pw[C] * zt[i] + zc;
        svp[i] = pw[C] * svp[i] + dpw[C] * sv[i] + spc;
        sv[i] = pw[C] * sv[i] + sc;
      }
    }
    zetap = pw[C] * zetap + dpw[C] * zeta + dgeo;
    zeta = pw[C] * zeta + geo;
    mma_wait_all(kMma, mph);
    if (tid == 0) {
      load(1, c + 1);
      load(2, c + 1);
    }
  }
  const float tot = block_sum(dl, red);
  if (tid == 0 && !*flag) atomicAdd(dlam + h, tot);
  if (tid == 0) {
    for (int b = 0; b < 4; ++b)
      for (int n = waited[b]; n < issued[b]; ++n) mbar_wait(bar(kFullQ + b), n & 1);
    umma_commit(bar(kFinal));
    mbar_wait(bar(kFinal), 0);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace btc
}  // namespace linattn
