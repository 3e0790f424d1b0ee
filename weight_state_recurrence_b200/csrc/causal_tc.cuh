// Chunked causal forward on the 5th-generation tensor cores (bf16 operands,
// fp32 accumulators in TMEM), d_k = 128, dv sliced 64 columns per CTA.
//
// The method (fast-weight article §2.1/§3.2/§4.2 recurrence, §3.1
// triangular-mask form, §4.1 note and §5.2 "cut the sequence into blocks:
// parallel inside a block, carried across blocks") written per chunk of
// C = 128 tokens, t and s 0-based inside the chunk, Cv valid tokens, state
// (S, z) carried from the previous chunk:
//
//   A        = (phi(Q) phi(K)^T) o M,   M[t][s] = lambda^(t-s) for s <= t, else 0
//   O        = A V  +  (Lq phi(Q)) S,                  Lq = diag(lambda^(t+1))
//   den      = rowsum(A) + (Lq phi(Q)) z + eps,        y = O / den
//   S       <- lambda^Cv S + (Lk phi(K))^T V,          Lk = diag(lambda^(Cv-1-t))
//   z       <- lambda^Cv z + (Lk phi(K))^T 1
//
// Every product above is one tcgen05.mma chain issued by a single thread:
//   A    : M=128 (t) x N=128 (s) x K=128 (d_k)   phi(Q) K-major, phi(K) K-major
//   O    : M=128 x N=64 x K=128 (s)              A (bf16, K-major) x V (MN-major)
//        + M=128 x N=64 x K=128 (d_k)            Lq phi(Q) (K-major) x S (bf16, MN-major)
//   qz   : M=128 x N=16 x K=128 (d_k)            Lq phi(Q) x [z_hi; z_lo; 0...] (K-major)
//   dS   : M=128 (d_k) x N=64 x K=128 (t)        (Lk phi(K))^T (MN-major) x V (MN-major)
//   dz   : M=128 (d_k) x N=16 x K=128 (t)        (Lk phi(K))^T x [1; 0...] (K-major)
// The fp32 state slice S (128 x 64) and z stay in registers of one
// warpgroup for the whole sequence; after each chunk they are re-emitted as
// bf16 operand tiles (z as a hi/lo bf16 pair so the denominator keeps ~16
// bits).  The denominator sums exactly the bf16-rounded weights that the
// numerator uses (row sums of the rounded A tile), so the output stays a
// normalised average.
//
// Decay powers lambda^i are formed directly per exponent (never as ratios),
// so lambda in [0, 1] including 0 is exact in form.
//
// Data movement: q, k, v tiles arrive by TMA (128B swizzle, out-of-range
// rows of a ragged last chunk read as zeros) into a two-stage ring; y leaves
// by TMA store from a swizzled staging tile (rows past N are clipped).
#pragma once
#include "common.cuh"
#include "sm100.cuh"

namespace linattn {
namespace tc {

constexpr int C = 128;      // tokens per chunk
constexpr int DK = 128;     // key dimension handled by this kernel
constexpr int DVS = 64;     // dv columns per CTA
constexpr int NT = 256;     // threads: warpgroup 0 = output side, warpgroup 1 = state side

constexpr uint32_t kPanel = C * 128;          // 128 rows x 128 bytes
constexpr uint32_t kOffQ = 0;                 // per stage: phi(Q), 2 panels (d_k 0-63, 64-127)
constexpr uint32_t kOffK = 2 * kPanel;        //            phi(K), 2 panels
constexpr uint32_t kOffV = 4 * kPanel;        //            V slice, 1 panel
constexpr uint32_t kStage = 5 * kPanel;
constexpr uint32_t kOffA = 2 * kStage;        // masked scores, 2 panels; later the y staging tile
constexpr uint32_t kOffS = kOffA + 2 * kPanel;  // S slice operand (bf16), 1 panel
constexpr uint32_t kOffZ = kOffS + kPanel;      // [z_hi; z_lo; 0..] 16 x 128, 2 panels of 2 KB
constexpr uint32_t kOffW = kOffZ + 4096;        // [1; 0..] 16 x 128, 2 panels of 2 KB
constexpr uint32_t kOffMisc = kOffW + 4096;     // barriers, TMEM slot, flags, decay table
constexpr uint32_t kMiscBytes = 2048;
constexpr uint32_t kSmemBytes = kOffMisc + kMiscBytes + 1024;  // + alignment slack
constexpr uint32_t kStageTxBytes = 5 * kPanel;

// TMEM columns (fp32, lane = row)
constexpr uint32_t kTmA = 0, kTmO = 128, kTmDS = 192, kTmQZ = 256, kTmDZ = 272;
constexpr uint32_t kTmCols = 512;

constexpr uint32_t kIdA = idesc_bf16(128, 128, 0, 0);
constexpr uint32_t kIdOV = idesc_bf16(128, 64, 0, 1);
constexpr uint32_t kIdOS = idesc_bf16(128, 64, 0, 1);
constexpr uint32_t kIdQZ = idesc_bf16(128, 16, 0, 0);
constexpr uint32_t kIdDS = idesc_bf16(128, 64, 1, 1);
constexpr uint32_t kIdDZ = idesc_bf16(128, 16, 1, 0);

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&p);
}

__device__ __forceinline__ float phi_fast(float x) { return x > 0.f ? x + 1.f : __expf(x); }

// phi applied in place to a bf16 tile (layout-agnostic: elementwise).
__device__ __forceinline__ void phi_tile_inplace(uint8_t *p, uint32_t bytes, int tid, int nthr) {
  for (uint32_t o = static_cast<uint32_t>(tid) * 16u; o < bytes; o += static_cast<uint32_t>(nthr) * 16u) {
    uint4 w = *reinterpret_cast<uint4 *>(p + o);
    uint32_t *u = reinterpret_cast<uint32_t *>(&w);
#pragma unroll
    for (int i = 0; i < 4; ++i) u[i] = pack_bf16(phi_fast(bf16lo(u[i])), phi_fast(bf16hi(u[i])));
    *reinterpret_cast<uint4 *>(p + o) = w;
  }
}

// Multiply every row r of a 2-panel swizzled tile (128 rows x 128 bf16) by
// scale[r] (rows keep their place under the swizzle: row = offset / 128).
__device__ __forceinline__ void scale_rows_inplace(uint8_t *p, const float *scale, int tid,
                                                   int nthr) {
  for (uint32_t o = static_cast<uint32_t>(tid) * 16u; o < 2 * kPanel;
       o += static_cast<uint32_t>(nthr) * 16u) {
    const float f = scale[(o % kPanel) >> 7];
    uint4 w = *reinterpret_cast<uint4 *>(p + o);
    uint32_t *u = reinterpret_cast<uint32_t *>(&w);
#pragma unroll
    for (int i = 0; i < 4; ++i) u[i] = pack_bf16(bf16lo(u[i]) * f, bf16hi(u[i]) * f);
    *reinterpret_cast<uint4 *>(p + o) = w;
  }
}

__global__ void __launch_bounds__(NT, 1)
    causal_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                     const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v,
                     const __grid_constant__ CUtensorMap tm_y, const float *__restrict__ lam,
                     float eps, float *__restrict__ S_final, float *__restrict__ z_final, int H,
                     int N, int DV) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                            ~static_cast<uintptr_t>(1023));
  const uint32_t sb = smem_u32(sm);
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int nslices = DV / DVS;
  const int pair = blockIdx.x / nslices;
  const int j0 = (blockIdx.x % nslices) * DVS;
  const int h = pair % H;
  const float L = lam ? lam[h] : 1.f;

  uint8_t *misc = sm + kOffMisc;
  const uint32_t bar_full0 = sb + kOffMisc + 0;   // stage 0 / 1 "data landed"
  const uint32_t bar_mma = sb + kOffMisc + 16;    // "issued MMAs complete"
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(misc + 32);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(misc + 36);
  float *pw = reinterpret_cast<float *>(misc + 64);     // lambda^i, i = 0..C
  float *qscale = pw + (C + 4);                         // lambda^(t+1)
  float *kscale = qscale + C;                           // lambda^(Cv-1-t), 0 past Cv

  if (tid == 0) {
    mbar_init(bar_full0, 1);
    mbar_init(bar_full0 + 8, 1);
    mbar_init(bar_mma, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_y);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), kTmCols);
    tmem_relinquish();
  }
  if (tid <= C) pw[tid] = pow_int(L, tid);
  // operand tiles that start as constants: S = 0, Z = 0, W = [1; 0...]
  for (uint32_t o = tid * 16u; o < kPanel; o += NT * 16u)
    *reinterpret_cast<uint4 *>(sm + kOffS + o) = make_uint4(0, 0, 0, 0);
  for (uint32_t o = tid * 16u; o < 4096u; o += NT * 16u) {
    *reinterpret_cast<uint4 *>(sm + kOffZ + o) = make_uint4(0, 0, 0, 0);
    const bool row0 = ((o % 2048u) >> 7) == 0;     // row 0 of either panel
    const uint32_t one2 = 0x3F803F80u;              // two bf16 ones
    *reinterpret_cast<uint4 *>(sm + kOffW + o) =
        row0 ? make_uint4(one2, one2, one2, one2) : make_uint4(0, 0, 0, 0);
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (tid <= C && tid >= 1) qscale[tid - 1] = pw[tid];
  const uint32_t tmem = *tmem_slot;

  const int nchunks = (N + C - 1) / C;
  auto issue_loads = [&](int c, int st) {
    const uint32_t base = sb + st * kStage;
    const uint32_t bar = bar_full0 + 8 * st;
    mbar_arrive_expect_tx(bar, kStageTxBytes);
    tma_load_3d(base + kOffQ, &tm_q, bar, 0, c * C, pair);
    tma_load_3d(base + kOffQ + kPanel, &tm_q, bar, 64, c * C, pair);
    tma_load_3d(base + kOffK, &tm_k, bar, 0, c * C, pair);
    tma_load_3d(base + kOffK + kPanel, &tm_k, bar, 64, c * C, pair);
    tma_load_3d(base + kOffV, &tm_v, bar, j0, c * C, pair);
  };
  if (tid == 0) {
    for (int c = 0; c < nchunks && c < 2; ++c) issue_loads(c, c);
  }

  // warpgroup-local indices: row owned by this thread and its TMEM lane field
  const int row = tid & 127;
  const uint32_t lane_field = static_cast<uint32_t>((warp & 3) * 32) << 16;
  float S_reg[DVS];
#pragma unroll
  for (int j = 0; j < DVS; ++j) S_reg[j] = 0.f;
  float z_reg = 0.f;
  float rowsum = 0.f;
  uint32_t mma_phase = 0;
  bool mma_in_flight = false;
  int next_consume = 0;                        // chunks [next_consume, next_issue) in flight
  int next_issue = nchunks < 2 ? nchunks : 2;

  for (int c = 0; c < nchunks; ++c) {
    const int st = c & 1;
    const uint32_t stage = sb + st * kStage;
    uint8_t *stage_p = sm + st * kStage;
    const int Cv = min(C, N - c * C);

    // ---- P1: inputs landed; apply phi in place to q and k
    if (!mbar_wait(bar_full0 + 8 * st, (c >> 1) & 1)) *abort_flag = 1;
    else next_consume = c + 1;
    if (tid < C) kscale[tid] = tid < Cv ? pw[Cv - 1 - tid] : 0.f;
    phi_tile_inplace(stage_p + kOffQ, 4 * kPanel, tid, NT);   // phi(Q) and phi(K) (adjacent)
    fence_proxy_async_smem();
    __syncthreads();
    if (*abort_flag) break;

    // ---- P2: A = phi(Q) phi(K)^T
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int ks = 0; ks < DK / 16; ++ks) {
        const uint32_t off = (ks >> 2) * kPanel + (ks & 3) * 32;
        umma_bf16(tmem + kTmA, sdesc_sw128(stage + kOffQ + off, 16, 1024),
                  sdesc_sw128(stage + kOffK + off, 16, 1024), kIdA, ks > 0);
      }
      umma_commit(bar_mma);
    }
    if (!mbar_wait(bar_mma, mma_phase)) {
      *abort_flag = 1;
      mma_in_flight = true;
    }
    mma_phase ^= 1;
    tc_fence_after();

    // ---- P3: warpgroup 0 masks/decays A into bf16; warpgroup 1 rescales Q and K rows
    if (warp < 4) {
      const int t = row;
      rowsum = 0.f;
#pragma unroll 1
      for (int blk = 0; blk < C / 32; ++blk) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(tmem + lane_field + kTmA + blk * 32, r);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int s0 = blk * 32 + 2 * i;
          const int e0 = t - s0, e1 = t - s0 - 1;
          const float f0 = (e0 >= 0 && s0 < Cv) ? pw[max(e0, 0)] : 0.f;
          const float f1 = (e1 >= 0 && s0 + 1 < Cv) ? pw[max(e1, 0)] : 0.f;
          pk[i] = pack_bf16(__uint_as_float(r[2 * i]) * f0, __uint_as_float(r[2 * i + 1]) * f1);
          rowsum += bf16lo(pk[i]) + bf16hi(pk[i]);
        }
        uint8_t *pa = sm + kOffA + (blk >> 1) * kPanel;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t byte = (blk & 1) * 64 + i * 16;
          *reinterpret_cast<uint4 *>(pa + sw128_offset(t, byte)) =
              make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
        }
      }
    } else {
      scale_rows_inplace(stage_p + kOffQ, qscale, tid - 128, 128);
      scale_rows_inplace(stage_p + kOffK, kscale, tid - 128, 128);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();

    // ---- P4: O = A V + (Lq phi(Q)) S ; qz ; dS ; dz
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int ks = 0; ks < C / 16; ++ks) {
        const uint32_t off = (ks >> 2) * kPanel + (ks & 3) * 32;
        umma_bf16(tmem + kTmO, sdesc_sw128(sb + kOffA + off, 16, 1024),
                  sdesc_sw128(stage + kOffV + ks * 2048, kPanel, 1024), kIdOV, ks > 0);
      }
#pragma unroll
      for (int ks = 0; ks < DK / 16; ++ks) {
        const uint32_t off = (ks >> 2) * kPanel + (ks & 3) * 32;
        umma_bf16(tmem + kTmO, sdesc_sw128(stage + kOffQ + off, 16, 1024),
                  sdesc_sw128(sb + kOffS + ks * 2048, kPanel, 1024), kIdOS, 1);
      }
#pragma unroll
      for (int ks = 0; ks < DK / 16; ++ks) {
        const uint32_t off = (ks >> 2) * kPanel + (ks & 3) * 32;
        const uint32_t offz = (ks >> 2) * 2048 + (ks & 3) * 32;
        umma_bf16(tmem + kTmQZ, sdesc_sw128(stage + kOffQ + off, 16, 1024),
                  sdesc_sw128(sb + kOffZ + offz, 16, 1024), kIdQZ, ks > 0);
      }
#pragma unroll
      for (int ks = 0; ks < C / 16; ++ks) {
        const uint64_t a = sdesc_sw128(stage + kOffK + ks * 2048, kPanel, 1024);
        umma_bf16(tmem + kTmDS, a, sdesc_sw128(stage + kOffV + ks * 2048, kPanel, 1024), kIdDS,
                  ks > 0);
        const uint32_t offw = (ks >> 2) * 2048 + (ks & 3) * 32;
        umma_bf16(tmem + kTmDZ, a, sdesc_sw128(sb + kOffW + offw, 16, 1024), kIdDZ, ks > 0);
      }
      umma_commit(bar_mma);
    }
    if (!mbar_wait(bar_mma, mma_phase)) {
      *abort_flag = 1;
      mma_in_flight = true;
    }
    mma_phase ^= 1;
    tc_fence_after();

    // ---- P5: warpgroup 0 writes y; warpgroup 1 advances the state
    if (warp < 4) {
      const int t = row;
      uint32_t o[64];
      uint32_t qz[2];
      tmem_ld_32x32b_x32(tmem + lane_field + kTmO, *reinterpret_cast<uint32_t(*)[32]>(&o[0]));
      tmem_ld_32x32b_x32(tmem + lane_field + kTmO + 32,
                         *reinterpret_cast<uint32_t(*)[32]>(&o[32]));
      tmem_ld_32x32b_x2(tmem + lane_field + kTmQZ, qz);
      tmem_wait_ld();
      const float inv = 1.f / (rowsum + (__uint_as_float(qz[0]) + __uint_as_float(qz[1])) + eps);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        uint4 w;
        w.x = pack_bf16(__uint_as_float(o[8 * i + 0]) * inv, __uint_as_float(o[8 * i + 1]) * inv);
        w.y = pack_bf16(__uint_as_float(o[8 * i + 2]) * inv, __uint_as_float(o[8 * i + 3]) * inv);
        w.z = pack_bf16(__uint_as_float(o[8 * i + 4]) * inv, __uint_as_float(o[8 * i + 5]) * inv);
        w.w = pack_bf16(__uint_as_float(o[8 * i + 6]) * inv, __uint_as_float(o[8 * i + 7]) * inv);
        *reinterpret_cast<uint4 *>(sm + kOffA + sw128_offset(t, i * 16)) = w;
      }
      fence_proxy_async_smem();
      named_bar_sync(1, 128);
      if (tid == 0) {
        tma_store_3d(&tm_y, sb + kOffA, j0, c * C, pair);
        tma_store_commit();
      }
    } else {
      const int kk = row;
      uint32_t d[64];
      uint32_t dz[2];
      tmem_ld_32x32b_x32(tmem + lane_field + kTmDS, *reinterpret_cast<uint32_t(*)[32]>(&d[0]));
      tmem_ld_32x32b_x32(tmem + lane_field + kTmDS + 32,
                         *reinterpret_cast<uint32_t(*)[32]>(&d[32]));
      tmem_ld_32x32b_x2(tmem + lane_field + kTmDZ, dz);
      tmem_wait_ld();
      const float g = pw[Cv];
#pragma unroll
      for (int j = 0; j < DVS; ++j) S_reg[j] = fmaf(g, S_reg[j], __uint_as_float(d[j]));
      z_reg = fmaf(g, z_reg, __uint_as_float(dz[0]));
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        uint4 w;
        w.x = pack_bf16(S_reg[8 * i + 0], S_reg[8 * i + 1]);
        w.y = pack_bf16(S_reg[8 * i + 2], S_reg[8 * i + 3]);
        w.z = pack_bf16(S_reg[8 * i + 4], S_reg[8 * i + 5]);
        w.w = pack_bf16(S_reg[8 * i + 6], S_reg[8 * i + 7]);
        *reinterpret_cast<uint4 *>(sm + kOffS + sw128_offset(kk, i * 16)) = w;
      }
      const __nv_bfloat16 zh = __float2bfloat16_rn(z_reg);
      const __nv_bfloat16 zl = __float2bfloat16_rn(z_reg - __bfloat162float(zh));
      const uint32_t zb = (kk >> 6) * 2048u;
      const uint32_t zbyte = (kk & 63) * 2;
      *reinterpret_cast<__nv_bfloat16 *>(sm + kOffZ + zb + sw128_offset(0, zbyte)) = zh;
      *reinterpret_cast<__nv_bfloat16 *>(sm + kOffZ + zb + sw128_offset(1, zbyte)) = zl;
      fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      if (c + 2 < nchunks) issue_loads(c + 2, st);
      tma_store_wait_read();   // the staging tile is rewritten by the next chunk's scores
    }
    __syncthreads();
    next_issue = min(nchunks, c + 3);
    if (*abort_flag) break;
  }

  if (*abort_flag) {
    // drain what this CTA still has in flight before releasing its resources
    // (each wait is bounded; a second time-out leaves the flag set)
    if (tid == 0) {
      for (int cc = next_consume; cc < next_issue; ++cc)
        mbar_wait(bar_full0 + 8 * (cc & 1), (cc >> 1) & 1);
      if (mma_in_flight) mbar_wait(bar_mma, mma_phase ^ 1);
    }
  } else if (warp >= 4) {
    const int kk = row;
    if (S_final) {
      float4 *dst = reinterpret_cast<float4 *>(S_final + (static_cast<long>(pair) * DK + kk) * DV + j0);
#pragma unroll
      for (int j = 0; j < DVS / 4; ++j)
        dst[j] = make_float4(S_reg[4 * j], S_reg[4 * j + 1], S_reg[4 * j + 2], S_reg[4 * j + 3]);
    }
    if (z_final && j0 == 0) z_final[static_cast<long>(pair) * DK + kk] = z_reg;
  }
  if (tid == 0) tma_store_wait_all();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmCols);
  }
}

}  // namespace tc
}  // namespace linattn
