// Global (non-causal) form on the tensor cores, d_k = d_v = 64, bf16:
//   KV = sum_n phi(k_n) v_n^T,  ksum = sum_n phi(k_n),
//   y_i = phi(q_i)^T KV / (phi(q_i)^T ksum + eps)
// (linear-attention note §3 after the sum swap and §6 forward; "Beyond
// self-attention", linear-attention code, here with eps).
//
// Two persistent kernels, each bound by HBM traffic (k and v are read once by
// the first, q read and y written once by the second):
//
// global_kv_tc_kernel: two heads of one sequence share every MMA (keys marked
//   as padding are zeroed with the feature map, so they enter neither sum).  With the
//   phi(k) tiles of both heads stacked along M (2 x 64 = 128 rows, MN-major)
//   and the v tiles side by side along N, D[128 x 128] += phi(K)^T V holds
//   both heads' KV on its diagonal blocks (the off-diagonal blocks are
//   discarded), and D2[128 x 16] += phi(K)^T 1 holds both ksum.  Each CTA
//   accumulates in TMEM over a contiguous range of 128-token chunks and adds
//   its partial sums into the caller's (zeroed) KV / ksum with vector fp32
//   reductions whenever its range leaves a head pair.
//
// global_out_tc_kernel: per 128-token tile of one head,
//   [O | qz_hi, qz_lo] = phi(Q) [KV | ksum_hi, ksum_lo]   (N = 80, K = 64)
//   with KV rounded to bf16 and ksum kept as a bf16 hi/lo pair, then
//   y = O / (qz + eps) stored by TMA from a swizzled staging tile.
//
// All barrier waits are bounded (sm100.cuh); the roles leave their loops
// together when one of them records a failure.
#pragma once
#include "common.cuh"
#include "sm100.cuh"

namespace linattn {
namespace gtc {

constexpr int C = 128;                 // tokens per tile
constexpr int D = 64;                  // d_k = d_v handled here
constexpr uint32_t kPanel = C * 128;   // one head's [128 tokens x 64] bf16 tile, 16 KB

__device__ __forceinline__ uint32_t pack2(float a, float b) {
  __nv_bfloat162 p = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&p);
}

__device__ __forceinline__ uint32_t phi2(uint32_t x) {
  const uint32_t zero = 0u, l2e_hi = 0x3FB93FB9u, l2e_lo = 0xBB2CBB2Cu;
  uint32_t m, r, t, e, y;
  asm("min.bf16x2 %0, %1, %2;" : "=r"(m) : "r"(x), "r"(zero));
  asm("max.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(x), "r"(zero));
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(t) : "r"(m), "r"(l2e_hi));
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(t) : "r"(m), "r"(l2e_lo), "r"(t));
  asm("ex2.approx.ftz.bf16x2 %0, %1;" : "=r"(e) : "r"(t));
  asm("add.rn.bf16x2 %0, %1, %2;" : "=r"(y) : "r"(r), "r"(e));
  return y;
}

// phi in place over `bytes` of swizzled tile rows (128 bytes per row); rows at
// or past `valid` become 0 when zero_tail (rows the TMA filled with zeros), and
// so do rows whose byte in `pad` (the tile's 128 rows of the key padding
// mask, or NULL) is nonzero.
__device__ __forceinline__ void phi_tile(uint8_t *p, uint32_t bytes, int valid, bool zero_tail,
                                         bool ident, int tid, int nthr,
                                         const uint8_t *pad = nullptr,
                                         uint32_t panel = kPanel) {
  const uint32_t step = static_cast<uint32_t>(nthr) * 16u;
  for (uint32_t o0 = static_cast<uint32_t>(tid) * 16u; o0 < bytes; o0 += 4 * step) {
    uint4 w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (o0 + i * step < bytes) w[i] = *reinterpret_cast<const uint4 *>(p + o0 + i * step);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t o = o0 + i * step;
      const int row = static_cast<int>((o % panel) >> 7);   // panels of `panel` bytes
      const bool dead = (zero_tail && row >= valid) || (pad && row < valid && pad[row]);
      w[i].x = dead ? 0u : ident ? w[i].x : phi2(w[i].x);
      w[i].y = dead ? 0u : ident ? w[i].y : phi2(w[i].y);
      w[i].z = dead ? 0u : ident ? w[i].z : phi2(w[i].z);
      w[i].w = dead ? 0u : ident ? w[i].w : phi2(w[i].w);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (o0 + i * step < bytes) *reinterpret_cast<uint4 *>(p + o0 + i * step) = w[i];
  }
}

__device__ __forceinline__ void red_add_v4(float *addr, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b),
               "f"(c), "f"(d)
               : "memory");
}

// Position (group, index) of a CTA's work unit u0 + i, for units laid out as
// groups of n consecutive indices, stepped one unit at a time: the loops need
// no 64-bit division per unit.
struct UnitCursor {
  int group, index, n;
  __device__ UnitCursor(long u0, int n_) : group(static_cast<int>(u0 / n_)),
                                           index(static_cast<int>(u0 % n_)), n(n_) {}
  __device__ void next() {
    if (++index == n) {
      index = 0;
      ++group;
    }
  }
};

// ============================================================= KV, ksum
namespace kv {
// Units of CK = 64 tokens of a head pair, so that the 3-deep ring (96 KB)
// leaves room for two CTAs per SM (80 registers a thread, 2 x 256 TMEM
// columns): one CTA's feature map and MMA chain overlap the other's.
constexpr int CK = 64;
constexpr uint32_t kPanelK = CK * 128;              // one head's [64 tokens x 64] bf16 tile, 8 KB
constexpr int kCtasPerSm = 2;
constexpr int kStages = 3;
constexpr uint32_t kStage = 4 * kPanelK;           // k head0, k head1, v head0, v head1
constexpr uint32_t kOffW = kStages * kStage;       // [1; 0 ...] 16 x 128 K-major, 2 x 2 KB
constexpr uint32_t kOffMisc = kOffW + 4096;
constexpr uint32_t kSmemBytes = kOffMisc + 512;
constexpr int NT = 384;                            // warp 0 TMA, 1 MMA, 4-11 phi + flush
constexpr int kXform = 256;
constexpr uint32_t kTmKV = 0, kTmKS = 128, kTmCols = 256;
enum { kFull = 0, kPhi = kStages, kEmpty = 2 * kStages, kFlushReady = 3 * kStages, kFlushDone,
       kFinal, kNumBars };
constexpr uint32_t kMiscTmem = 128, kMiscFail = 132, kMiscRoleFail = 136;
}  // namespace kv

__global__ void __launch_bounds__(kv::NT, kv::kCtasPerSm)
    global_kv_tc_kernel(const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v,
                        const uint8_t *__restrict__ kpm, float *__restrict__ KV,
                        float *__restrict__ ksum, int npairs, int N, int H, bool ident) {
  using namespace kv;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *sm = smem_raw;
  const uint32_t sb = smem_u32(sm);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (sb & 1023u) {
    if (tid == 0) atomicOr(&g_status, kStatusWaitTimeout);
    return;
  }
  auto bar = [&](int i) { return sb + kOffMisc + 8u * static_cast<uint32_t>(i); };
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + kOffMisc + kMiscTmem);
  volatile int *fail = reinterpret_cast<volatile int *>(sm + kOffMisc + kMiscFail);
  // set only before the role's named barrier, read only after it, so all
  // threads of the role take the same exit
  volatile int *rfail = reinterpret_cast<volatile int *>(sm + kOffMisc + kMiscRoleFail);

  const int nchunks = (N + CK - 1) / CK;
  const long units = static_cast<long>(npairs) * nchunks;
  const long u0 = units * blockIdx.x / gridDim.x, u1 = units * (blockIdx.x + 1) / gridDim.x;
  const int nmine = static_cast<int>(u1 - u0);

  if (tid == 0) {
    for (int i = 0; i < kNumBars; ++i) mbar_init(bar(i), 1);
    *fail = 0;
    *rfail = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmCols);
    tmem_relinquish();
  }
  for (uint32_t o = tid * 16u; o < 4096u; o += NT * 16u) {
    const bool row0 = ((o & 2047u) >> 7) == 0;
    const uint32_t one2 = 0x3F803F80u;
    *reinterpret_cast<uint4 *>(sm + kOffW + o) =
        row0 ? make_uint4(one2, one2, one2, one2) : make_uint4(0, 0, 0, 0);
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // the output kernel may start its CTAs on SMs this grid leaves (its q tiles
  // and phi(q) do not depend on KV; it waits for this grid before reading KV)
  grid_launch_dependents();
  // unit u0 + i of this CTA: pair (u0 + i) / nchunks, chunk (u0 + i) % nchunks,
  // tracked by a UnitCursor; a segment is a run of units of one pair, and the
  // accumulator is flushed at its end (the last unit, or the pair's last chunk)
  auto seg_end = [&](int i, const UnitCursor &u) { return i + 1 == nmine || u.index == nchunks - 1; };

  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;
      UnitCursor u(u0, nchunks);
      for (int i = 0; i < nmine && !*fail; ++i, u.next()) {
        const int s = i % kStages;
        if (i >= kStages && !mbar_wait(bar(kEmpty + s), ((i / kStages) - 1) & 1)) {
          *fail = 1;
          break;
        }
        const int p = u.group, c = u.index;
        const uint32_t st = sb + s * kStage, b = bar(kFull + s);
        mbar_arrive_expect_tx(b, kStage);
        tma_load_3d(st, &tm_k, b, 0, c * CK, 2 * p);
        tma_load_3d(st + kPanelK, &tm_k, b, 0, c * CK, 2 * p + 1);
        tma_load_3d(st + 2 * kPanelK, &tm_v, b, 0, c * CK, 2 * p);
        tma_load_3d(st + 3 * kPanelK, &tm_v, b, 0, c * CK, 2 * p + 1);
        issued = i + 1;
      }
      if (*fail)   // let the copies still in flight land before the CTA exits
        for (int i = issued - kStages < 0 ? 0 : issued - kStages; i < issued; ++i)
          mbar_wait(bar(kFull + i % kStages), (i / kStages) & 1);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idkv = idesc_bf16(128, 128, 1, 1), idks = idesc_bf16(128, 16, 1, 0);
      int seg = 0;
      bool first = true;
      UnitCursor u(u0, nchunks);
      for (int i = 0; i < nmine; ++i, u.next()) {
        const int s = i % kStages;
        if (*fail || !mbar_wait(bar(kPhi + s), (i / kStages) & 1)) {
          *fail = 1;
          break;
        }
        if (first && seg > 0 && !mbar_wait(bar(kFlushDone), (seg - 1) & 1)) {
          *fail = 1;
          break;
        }
        tc_fence_after();
        const uint32_t st = sb + s * kStage;
#pragma unroll
        for (int ks = 0; ks < CK / 16; ++ks) {
          // A = [phi(k) head0 | head1]^T: M = 128 (d_k of both heads), MN-major
          const uint64_t a = sdesc_sw128(st + ks * 2048, kPanelK, 1024);
          umma_bf16(tmem + kTmKV, a, sdesc_sw128(st + 2 * kPanelK + ks * 2048, kPanelK, 1024), idkv,
                    (!first || ks > 0) ? 1u : 0u);
          umma_bf16(tmem + kTmKS, a,
                    sdesc_sw128(sb + kOffW + (ks >> 2) * 2048 + (ks & 3) * 32, 16, 1024), idks,
                    (!first || ks > 0) ? 1u : 0u);
        }
        umma_commit(bar(kEmpty + s));
        first = false;
        if (seg_end(i, u)) {
          umma_commit(bar(kFlushReady));
          ++seg;
          first = true;
        }
      }
      umma_commit(bar(kFinal));
      mbar_wait(bar(kFinal), 0);
    }
    __syncwarp();
  } else if (warp >= 4) {
    const int tt = tid - 128;   // 0..255
    int seg = 0;
    UnitCursor u(u0, nchunks);
    for (int i = 0; i < nmine; ++i, u.next()) {
      const int s = i % kStages;
      if (*fail || !mbar_wait(bar(kFull + s), (i / kStages) & 1)) {
        *rfail = 1;
        *fail = 1;
      }
      const int valid = N - u.index * CK;
      // the pair's two heads belong to one sequence: one row of the padding mask
      const uint8_t *pad =
          kpm ? kpm + (2L * u.group / H) * N + static_cast<long>(u.index) * CK : nullptr;
      if (!*rfail)
        phi_tile(sm + s * kStage, 2 * kPanelK, valid, valid < CK, ident, tt, kXform, pad, kPanelK);
      fence_proxy_async_smem();
      named_bar_sync(1, kXform);
      if (*rfail) break;
      if (tt == 0) mbar_arrive(bar(kPhi + s));
      if (seg_end(i, u)) {
        // flush: lanes 0-63 are head 2p's d_k rows, 64-127 head 2p+1's.  The
        // verdict of the wait is shared through the barrier first, so that a
        // warp reads TMEM with all its lanes or not at all.
        const bool ok = !*fail && mbar_wait(bar(kFlushReady), seg & 1);
        if (!ok) {
          *rfail = 1;
          *fail = 1;
        }
        named_bar_sync(1, kXform);
        if (*rfail) break;
        tc_fence_after();
        if (warp < 8) {
          grid_dependency_wait();   // KV and ksum have been zeroed
          const int row = (warp - 4) * 32 + lane;
          const int hsel = row >> 6, kk = row & 63;
          const long bh = 2L * u.group + hsel;
          const uint32_t lf = static_cast<uint32_t>((warp - 4) * 32) << 16;
          uint32_t a[32], ksv[2];
          float *dst = KV + (bh * D + kk) * D;
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            tmem_ld_32x32b_x32(tmem + lf + kTmKV + hsel * 64 + half * 32, a);
            if (half == 0) tmem_ld_32x32b_x2(tmem + lf + kTmKS, ksv);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 8; ++j)
              red_add_v4(dst + half * 32 + 4 * j, __uint_as_float(a[4 * j]),
                         __uint_as_float(a[4 * j + 1]), __uint_as_float(a[4 * j + 2]),
                         __uint_as_float(a[4 * j + 3]));
            if (half == 0) atomicAdd(ksum + bh * D + kk, __uint_as_float(ksv[0]));
          }
        }
        tc_fence_before();
        named_bar_sync(1, kXform);
        if (*rfail) break;
        if (tt == 0) mbar_arrive(bar(kFlushDone));
        ++seg;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmCols);
  }
}

// ============================================================= outputs
namespace out {
constexpr int kStages = 4;
constexpr uint32_t kOffQ = 0;                           // kStages q tiles
constexpr uint32_t kOffB = kStages * kPanel;            // KV operand atom: 64 d_k rows x 64 cols
constexpr uint32_t kOffX = kOffB + 8192;                // [ksum_hi, ksum_lo, 0 ...] atom
constexpr uint32_t kOffY = kOffX + 8192;                // 2 y staging tiles
constexpr uint32_t kOffMisc = kOffY + 2 * kPanel;
constexpr uint32_t kSmemBytes = kOffMisc + 512;
constexpr int NT = 512;   // warp 0 TMA loads, 1 MMA, 2 TMA stores, 4-7 epilogue, 8-15 phi
// Two CTAs share an SM (64 registers a thread, 2 x 115.2 KB of shared memory,
// 2 x 256 TMEM columns), so one CTA's epilogue chain overlaps the other's.
constexpr int kCtasPerSm = 2;
constexpr int kXform = 256;
constexpr uint32_t kTmCols = 256;   // two 128-column accumulators (80 used each)
enum { kFull = 0, kPhi = kStages, kEmpty = 2 * kStages, kDFull = 3 * kStages, kDEmpty = kDFull + 2,
       kBReady = kDEmpty + 2, kYFull, kYFree = kYFull + 2, kFinal = kYFree + 2, kNumBars };
constexpr uint32_t kMiscTmem = 256, kMiscFail = 260, kMiscXFail = 264, kMiscEFail = 268;
}  // namespace out

__global__ void __launch_bounds__(out::NT, out::kCtasPerSm)
    global_out_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                         const __grid_constant__ CUtensorMap tm_y, const float *__restrict__ KV,
                         const float *__restrict__ ksum, float eps, int BH, int N,
                         bool ident) {
  using namespace out;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *sm = smem_raw;
  const uint32_t sb = smem_u32(sm);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (sb & 1023u) {
    if (tid == 0) atomicOr(&g_status, kStatusWaitTimeout);
    return;
  }
  auto bar = [&](int i) { return sb + kOffMisc + 8u * static_cast<uint32_t>(i); };
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + kOffMisc + kMiscTmem);
  volatile int *fail = reinterpret_cast<volatile int *>(sm + kOffMisc + kMiscFail);
  // per-role flags: written before the role's named barrier, read after it
  volatile int *xfail = reinterpret_cast<volatile int *>(sm + kOffMisc + kMiscXFail);
  volatile int *efail = reinterpret_cast<volatile int *>(sm + kOffMisc + kMiscEFail);

  const int ntiles = (N + C - 1) / C;
  const long units = static_cast<long>(BH) * ntiles;
  const long u0 = units * blockIdx.x / gridDim.x, u1 = units * (blockIdx.x + 1) / gridDim.x;
  const int nmine = static_cast<int>(u1 - u0);
  // unit u0 + i: head (u0 + i) / ntiles, tile (u0 + i) % ntiles, tracked by a
  // UnitCursor; a new head starts at the CTA's first unit or at tile 0
  auto seg_start = [&](int i, const UnitCursor &u) { return i == 0 || u.index == 0; };

  if (tid == 0) {
    for (int i = 0; i < kNumBars; ++i) mbar_init(bar(i), 1);
    *fail = 0;
    *xfail = 0;
    *efail = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_y);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmCols);
    tmem_relinquish();
  }
  for (uint32_t o = tid * 16u; o < 8192u; o += NT * 16u)
    *reinterpret_cast<uint4 *>(sm + kOffX + o) = make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;
      UnitCursor u(u0, ntiles);
      for (int i = 0; i < nmine && !*fail; ++i, u.next()) {
        const int s = i % kStages;
        if (i >= kStages && !mbar_wait(bar(kEmpty + s), ((i / kStages) - 1) & 1)) {
          *fail = 1;
          break;
        }
        const uint32_t b = bar(kFull + s);
        mbar_arrive_expect_tx(b, kPanel);
        tma_load_3d(sb + kOffQ + s * kPanel, &tm_q, b, 0, u.index * C, u.group);
        issued = i + 1;
      }
      if (*fail)   // let the copies still in flight land before the CTA exits
        for (int i = issued - kStages < 0 ? 0 : issued - kStages; i < issued; ++i)
          mbar_wait(bar(kFull + i % kStages), (i / kStages) & 1);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t id = idesc_bf16(128, 80, 0, 1);
      int seg = 0;
      UnitCursor u(u0, ntiles);
      for (int i = 0; i < nmine; ++i, u.next()) {
        const int s = i % kStages, d = i & 1;
        bool ok = !*fail && mbar_wait(bar(kPhi + s), (i / kStages) & 1);
        if (ok && seg_start(i, u)) ok = mbar_wait(bar(kBReady), seg++ & 1);
        if (ok && i >= 2) ok = mbar_wait(bar(kDEmpty + d), ((i >> 1) - 1) & 1);
        if (!ok) {
          *fail = 1;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks)
          umma_bf16(tmem + d * 128,
                    sdesc_sw128(sb + kOffQ + s * kPanel + ks * 32, 16, 1024),
                    sdesc_sw128(sb + kOffB + ks * 2048, kOffX - kOffB, 1024), id, ks > 0);
        umma_commit(bar(kDFull + d));
        umma_commit(bar(kEmpty + s));
      }
      umma_commit(bar(kFinal));
      mbar_wait(bar(kFinal), 0);
    }
    __syncwarp();
  } else if (warp == 2) {
    // y stores: issuing a 16 KB TMA store takes the issuing thread ~1 K
    // cycles, so it happens here, off the epilogue's per-tile chain.  Staging
    // tile d goes out once the epilogue has filled it, and is handed back once
    // the copy has read it.
    if (lane == 0) {
      UnitCursor u(u0, ntiles);
      for (int i = 0; i < nmine; ++i, u.next()) {
        const int d = i & 1;
        if (*fail || !mbar_wait(bar(kYFull + d), (i >> 1) & 1)) {
          *fail = 1;
          break;
        }
        tma_store_3d(&tm_y, sb + kOffY + d * kPanel, 0, u.index * C, u.group);
        tma_store_commit();
        tma_store_wait_read();
        mbar_arrive(bar(kYFree + d));
      }
      tma_store_wait_all();
    }
    __syncwarp();
  } else if (warp >= 8) {
    const int tt = tid - 256;
    for (int i = 0; i < nmine; ++i) {
      const int s = i % kStages;
      if (*fail || !mbar_wait(bar(kFull + s), (i / kStages) & 1)) {
        *xfail = 1;
        *fail = 1;
      }
      if (!*xfail && !ident) phi_tile(sm + kOffQ + s * kPanel, kPanel, C, false, false, tt, kXform);
      fence_proxy_async_smem();
      named_bar_sync(1, kXform);
      if (*xfail) break;
      if (tt == 0) mbar_arrive(bar(kPhi + s));
    }
  } else if (warp >= 4) {
    // epilogue warpgroup: (re)builds the [KV | ksum] operand at the start of
    // every head, then turns each accumulator tile into y
    const int r = (warp - 4) * 32 + lane;
    const uint32_t lf = static_cast<uint32_t>((warp - 4) * 32) << 16;
    UnitCursor u(u0, ntiles);
    for (int i = 0; i < nmine; ++i, u.next()) {
      const int d = i & 1;
      if (seg_start(i, u)) {
        // every earlier MMA has completed (its tile was consumed below), so
        // the operand can be rewritten: KV rows = d_k (K), 64 columns (N);
        // KV and ksum are complete once the KV grid has finished
        grid_dependency_wait();
        const long bh = u.group;
        if (r < D) {
          const float *src = KV + (bh * D + r) * D;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float4 a = *reinterpret_cast<const float4 *>(src + 8 * j);
            const float4 b = *reinterpret_cast<const float4 *>(src + 8 * j + 4);
            *reinterpret_cast<uint4 *>(sm + kOffB + sw128_offset(r, 16 * j)) =
                make_uint4(pack2(a.x, a.y), pack2(a.z, a.w), pack2(b.x, b.y), pack2(b.z, b.w));
          }
          const float kv = ksum[bh * D + r];
          const __nv_bfloat16 hi = __float2bfloat16_rn(kv);
          const __nv_bfloat16 lo = __float2bfloat16_rn(kv - __bfloat162float(hi));
          *reinterpret_cast<__nv_bfloat16 *>(sm + kOffX + sw128_offset(r, 0)) = hi;
          *reinterpret_cast<__nv_bfloat16 *>(sm + kOffX + sw128_offset(r, 2)) = lo;
        }
        fence_proxy_async_smem();
        named_bar_sync(2, 128);
        if (r == 0) mbar_arrive(bar(kBReady));
      }
      // every thread decides before the barrier and reads the verdict after
      // it, so the whole warpgroup takes the same path
      bool ok = !*fail && mbar_wait(bar(kDFull + d), (i >> 1) & 1);
      // staging tile d must be free: the store of tile i-2 has read it
      if (ok && i >= 2 && r == 0) ok = mbar_wait(bar(kYFree + d), ((i >> 1) - 1) & 1);
      if (!ok) {
        *efail = 1;
        *fail = 1;
      }
      tc_fence_after();
      named_bar_sync(2, 128);
      if (*efail) break;
      {
        uint32_t o[32], qz[2];
        tmem_ld_32x32b_x2(tmem + lf + d * 128 + 64, qz);
        tmem_ld_32x32b_x32(tmem + lf + d * 128, o);
        tmem_wait_ld();
        const float inv = 1.f / (__uint_as_float(qz[0]) + __uint_as_float(qz[1]) + eps);
        uint8_t *stg = sm + kOffY + d * kPanel;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          if (half == 1) {
            tmem_ld_32x32b_x32(tmem + lf + d * 128 + 32, o);
            tmem_wait_ld();
          }
#pragma unroll
          for (int j = 0; j < 4; ++j)
            *reinterpret_cast<uint4 *>(stg + sw128_offset(r, half * 64 + 16 * j)) = make_uint4(
                pack2(__uint_as_float(o[8 * j]) * inv, __uint_as_float(o[8 * j + 1]) * inv),
                pack2(__uint_as_float(o[8 * j + 2]) * inv, __uint_as_float(o[8 * j + 3]) * inv),
                pack2(__uint_as_float(o[8 * j + 4]) * inv, __uint_as_float(o[8 * j + 5]) * inv),
                pack2(__uint_as_float(o[8 * j + 6]) * inv, __uint_as_float(o[8 * j + 7]) * inv));
        }
      }
      tc_fence_before();
      fence_proxy_async_smem();
      named_bar_sync(2, 128);
      if (r == 0) {
        mbar_arrive(bar(kDEmpty + d));
        mbar_arrive(bar(kYFull + d));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmCols);
  }
}

// KV and ksum to zero before the KV kernel accumulates into them (one launch
// for both buffers; the KV kernel may start while this runs and waits for it
// only before its first flush)
__global__ void __launch_bounds__(256) zero2_kernel(float4 *__restrict__ a, long na4,
                                                    float4 *__restrict__ b, long nb4) {
  grid_launch_dependents();
  const long stride = static_cast<long>(gridDim.x) * blockDim.x;
  const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
  for (long i = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x; i < na4 + nb4; i += stride) {
    if (i < na4)
      a[i] = z;
    else
      b[i - na4] = z;
  }
}

}  // namespace gtc
}  // namespace linattn
