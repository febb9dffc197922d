// Backward pass, L side, on the tensor cores (bf16, T = 1; MonarchRT
// summary, "Method" (3): forward and backward kernels for finetuning with
// one refinement step).  The L side of the T = 1 forward is one softmax per
// query row (l, i) over the keys (k, q) of its row group p, with logits
// s = sc q . Kt + Hs, and O = L Y.  With G = dO its gradients are those of an
// attention with keys Kt, values Y and an additive bias:
//   dP = G Y^T,  delta = sum_{k,q} L dP (= G . O),  dS = L (dP - delta),
//   dq1 = sc dS Kt,  dKt = sc dS^T q,  dHs = column sums of dS,  dY = L^T G.
// One CTA of four warps per (g, i, p) when the row has at most 128 keys and
// the group at most 128 rows: q, dO, Kt and Y come in by TMA (128-byte
// swizzle), S and dP are two tcgen05 products into TMEM, one thread per row
// forms L and dS (bf16, shared memory, [row][key]), and three more products
// give dq1 (dS as the K-major A), [dKt | dHs] = dS^T [q | 1] and dY = L^T dO
// (dS^T and L^T as MN-major A operands, q and dO as MN-major B operands,
// with a block of ones appended to q for the column sums).
#include "bwd_tc.cuh"

#include <math.h>

#include <algorithm>
#include <mutex>

#include "tc_path.cuh"
#include "tc_ptx.cuh"
#include "timing.cuh"

namespace monarch {
namespace {

using namespace tc;

constexpr int kTile = 128;  // rows and keys of the tile = UMMA M = TMEM lanes
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct LBLayout {
  static constexpr int kChunk = kTile * 128;                   // 128 rows x 64 bf16, swizzled
  static constexpr int kQOff = 0;                              // D / 64 chunks, then ones
  static constexpr int kGOff = kQOff + (D / 64 + 1) * kChunk;  // dO
  static constexpr int kKtOff = kGOff + D / 64 * kChunk;       // Kt, 128 keys
  static constexpr int kYOff = kKtOff + D / 64 * kChunk;       // Y
  static constexpr int kLOff = kYOff + D / 64 * kChunk;        // L [row][key]: keys 0-63, 64-127
  static constexpr int kDSOff = kLOff + 2 * kChunk;            // dS [row][key]
  static constexpr int kBiasOff = kDSOff + 2 * kChunk;         // float [128]
  static constexpr int kBarOff = kBiasOff + kTile * 4;
  static constexpr int kBytes = kBarOff + 8 * 8;
  // TMEM: S [0, 128), dP [128, 256); then dq1 over S, dY over dP, and
  // [dKt | dHs] at [256, 256 + D + 64)
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kDPCol = 128, kDKCol = 256;
  static_assert(D == 64 || D == 128, "head dimension");
  static_assert(kBytes <= 227 * 1024, "shared memory");
};

struct LBArgs {
  const float* hs;  // [G][b2][c1][nk]
  float* dq1;       // [G][N][d]
  float* dkt;       // [G][b2][c1][nk][d]
  float* dy;
  float* dhs;       // [G][b2][c1][nk]
  bf16* dkt16;      // optional bf16 copies, [G][c1][nk][b2][d] (chunk-major)
  bf16* dy16;
  int b1, b2, c1, nk;
  float sc;
  int* status;
};

__device__ __forceinline__ void drain_bar(uint64_t* bar, uint32_t parity) {
  const unsigned long long t0 = global_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_ns() - t0 > kWaitLimitNs) break;
  }
}

// 16-byte unit u (keys 8u .. 8u + 7) of row r of a [row][key] bf16 tile of
// two 64-key chunks, 128-byte swizzled.
__device__ __forceinline__ uint4* rk_unit(uint8_t* tile, int r, int u) {
  return reinterpret_cast<uint4*>(tile + (u >> 3) * (kTile * 128) + r * 128 +
                                  (((u & 7) ^ (r & 7)) << 4));
}

template <int D>
__global__ void __launch_bounds__(128, 1)
    lbw_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_g,
               const __grid_constant__ CUtensorMap tm_kt, const __grid_constant__ CUtensorMap tm_y,
               LBArgs a) {
  using L = LBLayout<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5;
  if (smem_u32(smem) & 1023u) {  // swizzled tiles need 1024-B alignment: report, never fault
    if (tid == 0) atomicExch(a.status, 2);
    return;
  }
  int bid = blockIdx.x;
  const int p = bid % a.c1;
  bid /= a.c1;
  const int i = bid % a.b2;
  const int g = bid / a.b2;
  const int l0 = group_start(a.b1, a.c1, p), l1 = group_start(a.b1, a.c1, p + 1);
  const long key_row0 = ((long)(g * a.b2 + i) * a.c1 + p) * a.nk;
  uint8_t* sQ = smem + L::kQOff;
  uint8_t* sOnes = sQ + D / 64 * L::kChunk;
  uint8_t* sG = smem + L::kGOff;
  uint8_t* sKt = smem + L::kKtOff;
  uint8_t* sY = smem + L::kYOff;
  uint8_t* sL = smem + L::kLOff;
  uint8_t* sDS = smem + L::kDSOff;
  float* sBias = reinterpret_cast<float*>(smem + L::kBiasOff);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* load_full = bars + 0;
  uint64_t* s_full = bars + 1;
  uint64_t* o_full = bars + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 4);
  if (tid == 0) {
    mbar_init(load_full, 1);
    mbar_init(s_full, 1);
    mbar_init(o_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
  }
  for (int x = tid; x < L::kChunk / 16; x += 128)  // bf16 1.0 in every element
    reinterpret_cast<uint4*>(sOnes)[x] = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u,
                                                     0x3F803F80u);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
  bool issued_s = false, issued_o = false;
  if (tid == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_g);
    tma_prefetch_desc(&tm_kt);
    tma_prefetch_desc(&tm_y);
    mbar_arrive_expect_tx(load_full, 4 * (D / 64) * L::kChunk);
    // the 128 rows l0.. of position i (Monarch order: rows b2 d apart)
#pragma unroll
    for (int c = 0; c < D / 64; ++c) {
      tma_load_3d(sQ + c * L::kChunk, &tm_q, load_full, c * 64, i, g * a.b1 + l0);
      tma_load_3d(sG + c * L::kChunk, &tm_g, load_full, c * 64, i, g * a.b1 + l0);
      tma_load_2d(sKt + c * L::kChunk, &tm_kt, load_full, c * 64, (int)key_row0);
      tma_load_2d(sY + c * L::kChunk, &tm_y, load_full, c * 64, (int)key_row0);
    }
  }
  sBias[tid] = tid < a.nk ? a.hs[key_row0 + tid] : -INFINITY;
  __syncthreads();
  if (tid == 0 && mbar_wait(load_full, 0, abort_flag, a.status)) {
    tc_fence_after();
    const uint32_t idesc = idesc_bf16(kTile, kTile, false);
    const uint64_t dq = desc_kmajor(smem_u32(sQ)), dk = desc_kmajor(smem_u32(sKt));
    const uint64_t dg = desc_kmajor(smem_u32(sG)), dyd = desc_kmajor(smem_u32(sY));
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {  // S = q Kt^T
      const uint32_t off = ((kk >> 2) * L::kChunk + (kk & 3) * 32) >> 4;
      mma_bf16_ss(tmem, dq + off, dk + off, idesc, kk > 0 ? 1u : 0u);
    }
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {  // dP = dO Y^T
      const uint32_t off = ((kk >> 2) * L::kChunk + (kk & 3) * 32) >> 4;
      mma_bf16_ss(tmem + L::kDPCol, dg + off, dyd + off, idesc, kk > 0 ? 1u : 0u);
    }
    mma_commit(s_full);
    issued_s = true;
  }
  // ---- thread = row r of the group: L, delta, dS ----
  const int r = tid, l = l0 + r;
  const bool row_ok = l < l1;
  bool ok = mbar_wait(s_full, 0, abort_flag, a.status);
  ok = __syncthreads_and(ok);
  if (ok) {
    tc_fence_after();
    // the row's log-sum-exp over its keys (online over 32-key chunks)
    float m = -INFINITY, z = 0.f;
#pragma unroll 1
    for (int c = 0; c < kTile / 32; ++c) {
      float t[32];
      tmem_ld32(tmem + lane_off + c * 32, t);
      tmem_wait_ld();
      float mc = -INFINITY;
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        t[e] = fmaf(t[e], a.sc, sBias[c * 32 + e]);  // -inf past nk
        mc = fmaxf(mc, t[e]);
      }
      const float mn = fmaxf(m, mc);
      float zc = 0.f;
#pragma unroll
      for (int e = 0; e < 32; ++e) zc += ex2((t[e] - mn) * kLog2e);
      z = (m > -INFINITY ? z * ex2((m - mn) * kLog2e) : 0.f) + zc;
      m = mn;
    }
    const float lse2 = m * kLog2e + log2f(z);  // log2-units log-sum-exp
    // L = exp(s - lse) and delta = sum L dP; L (bf16) to its tile
    float delta = 0.f;
#pragma unroll 1
    for (int c = 0; c < kTile / 32; ++c) {
      float t[32], dp[32];
      tmem_ld32(tmem + lane_off + c * 32, t);
      tmem_ld32(tmem + lane_off + L::kDPCol + c * 32, dp);
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const float s = fmaf(t[e], a.sc, sBias[c * 32 + e]);
        t[e] = row_ok ? ex2(fmaf(s, kLog2e, -lse2)) : 0.f;
        delta = fmaf(t[e], dp[e], delta);
      }
#pragma unroll
      for (int uu = 0; uu < 4; ++uu) {
        const float* w = t + 8 * uu;
        uint4 pk;
        pk.x = pack_bf16x2(w[0], w[1]);
        pk.y = pack_bf16x2(w[2], w[3]);
        pk.z = pack_bf16x2(w[4], w[5]);
        pk.w = pack_bf16x2(w[6], w[7]);
        *rk_unit(sL, r, c * 4 + uu) = pk;
      }
    }
    // dS = L (dP - delta) (the same L, recomputed) to its tile
#pragma unroll 1
    for (int c = 0; c < kTile / 32; ++c) {
      float t[32], dp[32];
      tmem_ld32(tmem + lane_off + c * 32, t);
      tmem_ld32(tmem + lane_off + L::kDPCol + c * 32, dp);
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const float s = fmaf(t[e], a.sc, sBias[c * 32 + e]);
        const float w = row_ok ? ex2(fmaf(s, kLog2e, -lse2)) : 0.f;
        t[e] = w * (dp[e] - delta);
      }
#pragma unroll
      for (int uu = 0; uu < 4; ++uu) {
        const float* w = t + 8 * uu;
        uint4 pk;
        pk.x = pack_bf16x2(w[0], w[1]);
        pk.y = pack_bf16x2(w[2], w[3]);
        pk.z = pack_bf16x2(w[4], w[5]);
        pk.w = pack_bf16x2(w[6], w[7]);
        *rk_unit(sDS, r, c * 4 + uu) = pk;
      }
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  ok = __syncthreads_and(ok);
  if (ok && tid == 0) {
    tc_fence_after();
    // dq1~ = dS Kt: A = dS (rows x keys, K-major), B = Kt (keys x d, MN-major)
    {
      const uint32_t idesc = idesc_bf16(kTile, D, true);
      const uint64_t da = desc_kmajor(smem_u32(sDS));
      const uint64_t db = desc_mnmajor(smem_u32(sKt), L::kChunk);
#pragma unroll
      for (int kk = 0; kk < kTile / 16; ++kk)
        mma_bf16_ss(tmem, da + (((kk >> 2) * L::kChunk + (kk & 3) * 32) >> 4),
                    db + ((kk * 16 * 128) >> 4), idesc, kk > 0 ? 1u : 0u);
    }
    // [dKt~ | dHs] = dS^T [q | 1] and dY = L^T dO: A MN-major (keys
    // contiguous in each row), B MN-major (d contiguous in each row)
    {
      const uint32_t idesc_k = idesc_bf16(kTile, D + 64, true, true);
      const uint32_t idesc_y = idesc_bf16(kTile, D, true, true);
      const uint64_t ds = desc_mnmajor(smem_u32(sDS), L::kChunk);
      const uint64_t lw = desc_mnmajor(smem_u32(sL), L::kChunk);
      const uint64_t qb = desc_mnmajor(smem_u32(sQ), L::kChunk);
      const uint64_t gb = desc_mnmajor(smem_u32(sG), L::kChunk);
#pragma unroll
      for (int kk = 0; kk < kTile / 16; ++kk) {
        const uint32_t off = (kk * 16 * 128) >> 4;
        mma_bf16_ss(tmem + L::kDKCol, ds + off, qb + off, idesc_k, kk > 0 ? 1u : 0u);
        mma_bf16_ss(tmem + L::kDPCol, lw + off, gb + off, idesc_y, kk > 0 ? 1u : 0u);
      }
    }
    mma_commit(o_full);
    issued_o = true;
  }
  if (ok) ok = mbar_wait(o_full, 0, abort_flag, a.status);
  ok = __syncthreads_and(ok);
  if (ok) {
    tc_fence_after();
    // thread = row: dq1 (rows of the group only)
    float* dqrow = a.dq1 + ((long)(g * a.b1 + l) * a.b2 + i) * D;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      float t[32];
      tmem_ld32(tmem + lane_off + c * 32, t);
      tmem_wait_ld();
      if (row_ok) {
#pragma unroll
        for (int e = 0; e < 32; e += 4)
          *reinterpret_cast<float4*>(dqrow + c * 32 + e) =
              make_float4(t[e] * a.sc, t[e + 1] * a.sc, t[e + 2] * a.sc, t[e + 3] * a.sc);
      }
    }
    // thread = key m: dKt, dHs, dY
    const int m = tid;
    const bool key_ok = m < a.nk;
    float* dkrow = a.dkt + (key_row0 + m) * D;
    float* dyrow = a.dy + (key_row0 + m) * D;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      float t[32], u[32];
      tmem_ld32(tmem + lane_off + L::kDKCol + c * 32, t);
      tmem_ld32(tmem + lane_off + L::kDPCol + c * 32, u);
      tmem_wait_ld();
      if (key_ok) {
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          *reinterpret_cast<float4*>(dkrow + c * 32 + e) =
              make_float4(t[e] * a.sc, t[e + 1] * a.sc, t[e + 2] * a.sc, t[e + 3] * a.sc);
          *reinterpret_cast<float4*>(dyrow + c * 32 + e) =
              make_float4(u[e], u[e + 1], u[e + 2], u[e + 3]);
        }
        if (a.dkt16 != nullptr) {
          const long crow = (((long)g * a.c1 + p) * a.nk + m) * a.b2 + i;
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            uint4 pk, pv;
            pk.x = pack_bf16x2(t[e] * a.sc, t[e + 1] * a.sc);
            pk.y = pack_bf16x2(t[e + 2] * a.sc, t[e + 3] * a.sc);
            pk.z = pack_bf16x2(t[e + 4] * a.sc, t[e + 5] * a.sc);
            pk.w = pack_bf16x2(t[e + 6] * a.sc, t[e + 7] * a.sc);
            pv.x = pack_bf16x2(u[e], u[e + 1]);
            pv.y = pack_bf16x2(u[e + 2], u[e + 3]);
            pv.z = pack_bf16x2(u[e + 4], u[e + 5]);
            pv.w = pack_bf16x2(u[e + 6], u[e + 7]);
            *reinterpret_cast<uint4*>(a.dkt16 + crow * D + c * 32 + e) = pk;
            *reinterpret_cast<uint4*>(a.dy16 + crow * D + c * 32 + e) = pv;
          }
        }
      }
    }
    float cs[32];
    tmem_ld32(tmem + lane_off + L::kDKCol + D, cs);
    tmem_wait_ld();
    if (key_ok) a.dhs[key_row0 + m] = cs[0];
  }
  if (tid == 0 && *abort_flag) {  // drain what this CTA issued (bounded)
    if (!issued_s) drain_bar(load_full, 0);
    if (issued_s) drain_bar(s_full, 0);
    if (issued_o) drain_bar(o_full, 0);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// R side of the backward, untiled (c1 = c2 = 1, b2 <= 128): one CTA of four
// warps per chunk (g, k), rows i = the b2 positions, keys j = the chunk's b2
// keys.  With the L side's dKt, dY (bf16, chunk-major) and dHs:
//   S_R = sc Qt0 K^T,  R = softmax_j S_R,
//   dR = dKt K^T + dY V^T - dHs (ln R + 1),  dS_R = R (dR - sum_j R dR),
//   partial dQt0 = sc dS_R K,  dk = R^T dKt + sc dS_R^T Qt0,  dv = R^T dY
// (the chain rule through Kt = R K, Y = R V and Hs = the entropy of R).  S_R
// and dR are products into TMEM; one thread per row forms R and sc dS_R
// (bf16, [row][key]); the three gradients are products with R^T and dS_R^T
// as MN-major A operands.
// ---------------------------------------------------------------------------
template <int D>
struct RBLayout {
  static constexpr int kChunk = kTile * 128;
  static constexpr int kQOff = 0;                          // Qt0 rows i
  static constexpr int kKOff = kQOff + D / 64 * kChunk;    // K rows j
  static constexpr int kVOff = kKOff + D / 64 * kChunk;    // V rows j
  static constexpr int kDKOff = kVOff + D / 64 * kChunk;   // dKt rows i
  static constexpr int kDYOff = kDKOff + D / 64 * kChunk;  // dY rows i
  static constexpr int kROff = kDYOff + D / 64 * kChunk;   // R [i][j]: keys 0-63, 64-127
  static constexpr int kDSOff = kROff + 2 * kChunk;        // sc dS_R [i][j]
  static constexpr int kBarOff = kDSOff + 2 * kChunk;
  static constexpr int kBytes = kBarOff + 8 * 8;
  // TMEM: S_R [0, 128), dR [128, 256); then partial dQt0 over S_R, dv over
  // dR, dk at [256, 256 + D)
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kDRCol = 128, kDKCol = 256;
  static_assert(D == 64 || D == 128, "head dimension");
  static_assert(kBytes <= 227 * 1024, "shared memory");
};

struct RBArgs {
  const float* dhs;  // [G][b2 i][b1 k]
  float* dqt0_part;  // [G][b2 i][b1 k][d]
  bf16* dk;          // (G, N, d)
  bf16* dv;
  int b1, b2;
  float sc;
  int* status;
};

template <int D>
__global__ void __launch_bounds__(128, 1)
    rbw_kernel(const __grid_constant__ CUtensorMap tm_qt0, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_dk,
               const __grid_constant__ CUtensorMap tm_dy, RBArgs a) {
  using L = RBLayout<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5;
  if (smem_u32(smem) & 1023u) {
    if (tid == 0) atomicExch(a.status, 2);
    return;
  }
  const int k = blockIdx.x % a.b1;
  const int g = blockIdx.x / a.b1;
  const int chunk_row0 = (g * a.b1 + k) * a.b2;  // keys j of chunk k; dKt, dY rows i of (g, k)
  uint8_t* sQ = smem + L::kQOff;
  uint8_t* sK = smem + L::kKOff;
  uint8_t* sV = smem + L::kVOff;
  uint8_t* sDK = smem + L::kDKOff;
  uint8_t* sDY = smem + L::kDYOff;
  uint8_t* sR = smem + L::kROff;
  uint8_t* sDS = smem + L::kDSOff;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* load_full = bars + 0;
  uint64_t* s_full = bars + 1;
  uint64_t* o_full = bars + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 4);
  if (tid == 0) {
    mbar_init(load_full, 1);
    mbar_init(s_full, 1);
    mbar_init(o_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
  bool issued_s = false, issued_o = false;
  if (tid == 0) {
    tma_prefetch_desc(&tm_qt0);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_dk);
    tma_prefetch_desc(&tm_dy);
    mbar_arrive_expect_tx(load_full, 5 * (D / 64) * L::kChunk);
#pragma unroll
    for (int c = 0; c < D / 64; ++c) {
      tma_load_2d(sQ + c * L::kChunk, &tm_qt0, load_full, c * 64, g * a.b2);
      tma_load_2d(sK + c * L::kChunk, &tm_k, load_full, c * 64, chunk_row0);
      tma_load_2d(sV + c * L::kChunk, &tm_v, load_full, c * 64, chunk_row0);
      tma_load_2d(sDK + c * L::kChunk, &tm_dk, load_full, c * 64, chunk_row0);
      tma_load_2d(sDY + c * L::kChunk, &tm_dy, load_full, c * 64, chunk_row0);
    }
    if (mbar_wait(load_full, 0, abort_flag, a.status)) {
      tc_fence_after();
      const uint32_t idesc = idesc_bf16(kTile, kTile, false);
      const uint64_t dq = desc_kmajor(smem_u32(sQ)), dkk = desc_kmajor(smem_u32(sK));
      const uint64_t dvv = desc_kmajor(smem_u32(sV)), ddk = desc_kmajor(smem_u32(sDK));
      const uint64_t ddy = desc_kmajor(smem_u32(sDY));
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {  // S_R / sc = Qt0 K^T
        const uint32_t off = ((kk >> 2) * L::kChunk + (kk & 3) * 32) >> 4;
        mma_bf16_ss(tmem, dq + off, dkk + off, idesc, kk > 0 ? 1u : 0u);
      }
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {  // dKt K^T
        const uint32_t off = ((kk >> 2) * L::kChunk + (kk & 3) * 32) >> 4;
        mma_bf16_ss(tmem + L::kDRCol, ddk + off, dkk + off, idesc, kk > 0 ? 1u : 0u);
      }
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {  // + dY V^T
        const uint32_t off = ((kk >> 2) * L::kChunk + (kk & 3) * 32) >> 4;
        mma_bf16_ss(tmem + L::kDRCol, ddy + off, dvv + off, idesc, 1u);
      }
      mma_commit(s_full);
      issued_s = true;
    }
  }
  // ---- thread = row i: R, dR, sc dS_R ----
  const int r = tid;
  const bool row_ok = r < a.b2;
  bool ok = mbar_wait(s_full, 0, abort_flag, a.status);
  ok = __syncthreads_and(ok);
  if (ok) {
    tc_fence_after();
    const float s2 = a.sc * kLog2e;  // logits in log2 units
    float m = -INFINITY;
#pragma unroll 1
    for (int c = 0; c < kTile / 32; ++c) {
      float t[32];
      tmem_ld32(tmem + lane_off + c * 32, t);
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 32; ++e)
        if (c * 32 + e < a.b2) m = fmaxf(m, t[e] * s2);
    }
    float z = 0.f;
#pragma unroll 1
    for (int c = 0; c < kTile / 32; ++c) {
      float t[32];
      tmem_ld32(tmem + lane_off + c * 32, t);
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 32; ++e)
        if (c * 32 + e < a.b2) z += ex2(fmaf(t[e], s2, -m));
    }
    const float lz = m + log2f(z);  // log2 of the row's normaliser
    const float dh = row_ok ? a.dhs[((long)g * a.b2 + r) * a.b1 + k] : 0.f;
    // rho = sum_j R dR, with dR including the entropy term; R to its tile
    float rho = 0.f;
#pragma unroll 1
    for (int c = 0; c < kTile / 32; ++c) {
      float t[32], dr[32];
      tmem_ld32(tmem + lane_off + c * 32, t);
      tmem_ld32(tmem + lane_off + L::kDRCol + c * 32, dr);
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const float x2 = fmaf(t[e], s2, -lz);  // log2 R
        const bool live = row_ok && c * 32 + e < a.b2;
        const float w = live ? ex2(x2) : 0.f;
        const float d_r = dr[e] - dh * (x2 * 0.69314718055994531f + 1.f);
        rho = fmaf(w, live ? d_r : 0.f, rho);
        t[e] = w;
      }
#pragma unroll
      for (int uu = 0; uu < 4; ++uu) {
        const float* w = t + 8 * uu;
        uint4 pk;
        pk.x = pack_bf16x2(w[0], w[1]);
        pk.y = pack_bf16x2(w[2], w[3]);
        pk.z = pack_bf16x2(w[4], w[5]);
        pk.w = pack_bf16x2(w[6], w[7]);
        *rk_unit(sR, r, c * 4 + uu) = pk;
      }
    }
#pragma unroll 1
    for (int c = 0; c < kTile / 32; ++c) {
      float t[32], dr[32];
      tmem_ld32(tmem + lane_off + c * 32, t);
      tmem_ld32(tmem + lane_off + L::kDRCol + c * 32, dr);
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const float x2 = fmaf(t[e], s2, -lz);
        const bool live = row_ok && c * 32 + e < a.b2;
        const float w = live ? ex2(x2) : 0.f;
        const float d_r = dr[e] - dh * (x2 * 0.69314718055994531f + 1.f);
        t[e] = live ? a.sc * w * (d_r - rho) : 0.f;
      }
#pragma unroll
      for (int uu = 0; uu < 4; ++uu) {
        const float* w = t + 8 * uu;
        uint4 pk;
        pk.x = pack_bf16x2(w[0], w[1]);
        pk.y = pack_bf16x2(w[2], w[3]);
        pk.z = pack_bf16x2(w[4], w[5]);
        pk.w = pack_bf16x2(w[6], w[7]);
        *rk_unit(sDS, r, c * 4 + uu) = pk;
      }
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  ok = __syncthreads_and(ok);
  if (ok && tid == 0) {
    tc_fence_after();
    // partial dQt0 = (sc dS_R) K: A K-major (rows x keys), B = K MN-major
    {
      const uint32_t idesc = idesc_bf16(kTile, D, true);
      const uint64_t da = desc_kmajor(smem_u32(sDS));
      const uint64_t db = desc_mnmajor(smem_u32(sK), L::kChunk);
#pragma unroll
      for (int kk = 0; kk < kTile / 16; ++kk)
        mma_bf16_ss(tmem, da + (((kk >> 2) * L::kChunk + (kk & 3) * 32) >> 4),
                    db + ((kk * 16 * 128) >> 4), idesc, kk > 0 ? 1u : 0u);
    }
    // dk = R^T dKt + (sc dS_R)^T Qt0 and dv = R^T dY: A MN-major (keys
    // contiguous in each row), B MN-major (d contiguous in each row)
    {
      const uint32_t idesc = idesc_bf16(kTile, D, true, true);
      const uint64_t rw = desc_mnmajor(smem_u32(sR), L::kChunk);
      const uint64_t ds = desc_mnmajor(smem_u32(sDS), L::kChunk);
      const uint64_t bdk = desc_mnmajor(smem_u32(sDK), L::kChunk);
      const uint64_t bq = desc_mnmajor(smem_u32(sQ), L::kChunk);
      const uint64_t bdy = desc_mnmajor(smem_u32(sDY), L::kChunk);
#pragma unroll
      for (int kk = 0; kk < kTile / 16; ++kk) {
        const uint32_t off = (kk * 16 * 128) >> 4;
        mma_bf16_ss(tmem + L::kDKCol, rw + off, bdk + off, idesc, kk > 0 ? 1u : 0u);
      }
#pragma unroll
      for (int kk = 0; kk < kTile / 16; ++kk) {
        const uint32_t off = (kk * 16 * 128) >> 4;
        mma_bf16_ss(tmem + L::kDKCol, ds + off, bq + off, idesc, 1u);
      }
#pragma unroll
      for (int kk = 0; kk < kTile / 16; ++kk) {
        const uint32_t off = (kk * 16 * 128) >> 4;
        mma_bf16_ss(tmem + L::kDRCol, rw + off, bdy + off, idesc, kk > 0 ? 1u : 0u);
      }
    }
    mma_commit(o_full);
    issued_o = true;
  }
  if (ok) ok = mbar_wait(o_full, 0, abort_flag, a.status);
  ok = __syncthreads_and(ok);
  if (ok) {
    tc_fence_after();
    // thread = row i: the partial dQt0 of (g, i, k)
    float* prow = a.dqt0_part + (((long)g * a.b2 + r) * a.b1 + k) * D;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      float t[32];
      tmem_ld32(tmem + lane_off + c * 32, t);
      tmem_wait_ld();
      if (row_ok) {
#pragma unroll
        for (int e = 0; e < 32; e += 4)
          *reinterpret_cast<float4*>(prow + c * 32 + e) =
              make_float4(t[e], t[e + 1], t[e + 2], t[e + 3]);
      }
    }
    // thread = key j: dk and dv of token k b2 + j
    const bool key_ok = tid < a.b2;
    bf16* dkrow = a.dk + ((long)chunk_row0 + tid) * D;
    bf16* dvrow = a.dv + ((long)chunk_row0 + tid) * D;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      float t[32], u[32];
      tmem_ld32(tmem + lane_off + L::kDKCol + c * 32, t);
      tmem_ld32(tmem + lane_off + L::kDRCol + c * 32, u);
      tmem_wait_ld();
      if (key_ok) {
#pragma unroll
        for (int e = 0; e < 32; e += 8) {
          uint4 pk, pv;
          pk.x = pack_bf16x2(t[e], t[e + 1]);
          pk.y = pack_bf16x2(t[e + 2], t[e + 3]);
          pk.z = pack_bf16x2(t[e + 4], t[e + 5]);
          pk.w = pack_bf16x2(t[e + 6], t[e + 7]);
          pv.x = pack_bf16x2(u[e], u[e + 1]);
          pv.y = pack_bf16x2(u[e + 2], u[e + 3]);
          pv.z = pack_bf16x2(u[e + 4], u[e + 5]);
          pv.w = pack_bf16x2(u[e + 6], u[e + 7]);
          *reinterpret_cast<uint4*>(dkrow + c * 32 + e) = pk;
          *reinterpret_cast<uint4*>(dvrow + c * 32 + e) = pv;
        }
      }
    }
  }
  if (tid == 0 && *abort_flag) {  // drain what this CTA issued (bounded)
    if (!issued_s) drain_bar(load_full, 0);
    if (issued_s) drain_bar(s_full, 0);
    if (issued_o) drain_bar(o_full, 0);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

template <int D>
cudaError_t launch_rbw(const bf16* qt0_16, const bf16* k, const bf16* v, const bf16* dkt16,
                       const bf16* dy16, const float* dhs, float* dqt0_part, bf16* dk, bf16* dv,
                       const Problem& pb, int* status, cudaStream_t stream, int* launches) {
  using L = RBLayout<D>;
  static std::once_flag attr_once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(attr_once, [] {
    attr_err = cudaFuncSetAttribute(rbw_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    L::kBytes);
  });
  if (attr_err != cudaSuccess) return attr_err;
  const long n_rows = (long)pb.G * pb.b1 * pb.b2;  // tokens, and rows of dKt / dY per head
  CUtensorMap tq, tk, tv, tdk, tdy;
  const cuuint64_t str[1] = {(cuuint64_t)D * 2};
  const cuuint32_t box[2] = {64, kTile};
  {
    const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)pb.G * pb.b2};
    if (!tc_make_map(&tq, qt0_16, 2, dims, str, box)) return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)n_rows};
    if (!tc_make_map(&tk, k, 2, dims, str, box) || !tc_make_map(&tv, v, 2, dims, str, box) ||
        !tc_make_map(&tdk, dkt16, 2, dims, str, box) || !tc_make_map(&tdy, dy16, 2, dims, str, box))
      return cudaErrorInvalidValue;
  }
  RBArgs a;
  a.dhs = dhs;
  a.dqt0_part = dqt0_part;
  a.dk = dk;
  a.dv = dv;
  a.b1 = pb.b1;
  a.b2 = pb.b2;
  a.sc = pb.sc;
  a.status = status;
  return timed_launch("bwd_tc_r_side", stream, launches, [&] {
    rbw_kernel<D><<<(unsigned)((long)pb.G * pb.b1), 128, L::kBytes, stream>>>(tq, tk, tv, tdk,
                                                                               tdy, a);
  });
}

// bf16 -> fp32 of n elements.
__global__ void to_f32_kernel(const bf16* __restrict__ a, float* __restrict__ out, long n) {
  for (long x = blockIdx.x * (long)blockDim.x + threadIdx.x; x < n;
       x += (long)gridDim.x * blockDim.x)
    out[x] = __bfloat162float(a[x]);
}

template <int D>
cudaError_t launch_lbw(const bf16* q, const bf16* dout, const bf16* kt16, const bf16* y16,
                       const float* hs, float* dq1, float* dkt, float* dy, float* dhs,
                       bf16* dkt16, bf16* dy16, const Problem& pb, int* status,
                       cudaStream_t stream, int* launches) {
  using L = LBLayout<D>;
  static std::once_flag attr_once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(attr_once, [] {
    attr_err = cudaFuncSetAttribute(lbw_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    L::kBytes);
  });
  if (attr_err != cudaSuccess) return attr_err;
  const int nk = pb.b1 * pb.c2;
  const long key_rows = (long)pb.G * pb.b2 * pb.c1 * nk;
  CUtensorMap tq, tg, tk, ty;
  if (!tc_make_q_slab_map(&tq, q, pb, D) || !tc_make_q_slab_map(&tg, dout, pb, D))
    return cudaErrorInvalidValue;
  {
    const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)key_rows};
    const cuuint64_t str[1] = {(cuuint64_t)D * 2};
    const cuuint32_t box[2] = {64, kTile};
    if (!tc_make_map(&tk, kt16, 2, dims, str, box) || !tc_make_map(&ty, y16, 2, dims, str, box))
      return cudaErrorInvalidValue;
  }
  LBArgs a;
  a.hs = hs;
  a.dq1 = dq1;
  a.dkt = dkt;
  a.dy = dy;
  a.dhs = dhs;
  a.dkt16 = dkt16;
  a.dy16 = dy16;
  a.b1 = pb.b1;
  a.b2 = pb.b2;
  a.c1 = pb.c1;
  a.nk = nk;
  a.sc = pb.sc;
  a.status = status;
  const long blocks = (long)pb.G * pb.b2 * pb.c1;
  return timed_launch("bwd_tc_l_side", stream, launches, [&] {
    lbw_kernel<D><<<(unsigned)blocks, 128, L::kBytes, stream>>>(tq, tg, tk, ty, a);
  });
}

}  // namespace

bool bwd_tc_l_side_supports(const Problem& pb) {
  if (pb.d != 64 && pb.d != 128) return false;
  if (pb.tr || is_padded(pb) || pb.T != 1 || !tc_supports(pb)) return false;
  if (pb.b1 * pb.c2 > kTile || (pb.b1 + pb.c1 - 1) / pb.c1 > kTile) return false;
  const long key_rows = (long)pb.G * pb.b2 * pb.c1 * pb.b1 * pb.c2;
  return key_rows + kTile < (1L << 31) && (long)pb.G * pb.b1 < (1L << 31);
}

cudaError_t bwd_tc_recompute(const bf16* q, const bf16* k, const bf16* v, bf16* qt0_16,
                             bf16* kt16, bf16* y16, float* hs, float* qt0, const Problem& pb,
                             int* status, cudaStream_t stream, int* launches) {
  if (!bwd_tc_l_side_supports(pb)) return cudaErrorInvalidValue;
  cudaError_t e = tc_step_one(q, k, v, qt0_16, kt16, y16, hs, pb, status, stream, launches);
  if (e != cudaSuccess) return e;
  const long n = (long)pb.G * pb.c1 * pb.b2 * pb.d;
  return timed_launch("bwd_tc_qt0_f32", stream, launches, [&] {
    to_f32_kernel<<<(unsigned)std::min<long>((n + 255) / 256, 148L * 8), 256, 0, stream>>>(
        qt0_16, qt0, n);
  });
}

cudaError_t bwd_tc_l_side(const bf16* q, const bf16* dout, const bf16* kt16, const bf16* y16,
                          const float* hs, float* dq1, float* dkt, float* dy, float* dhs,
                          bf16* dkt16, bf16* dy16, const Problem& pb, int* status,
                          cudaStream_t stream, int* launches) {
  if (!bwd_tc_l_side_supports(pb)) return cudaErrorInvalidValue;
  return pb.d == 128 ? launch_lbw<128>(q, dout, kt16, y16, hs, dq1, dkt, dy, dhs, dkt16, dy16, pb,
                                       status, stream, launches)
                     : launch_lbw<64>(q, dout, kt16, y16, hs, dq1, dkt, dy, dhs, dkt16, dy16, pb,
                                      status, stream, launches);
}

bool bwd_tc_r_side_supports(const Problem& pb) {
  return bwd_tc_l_side_supports(pb) && pb.c1 == 1 && pb.c2 == 1 && pb.b2 <= kTile;
}

cudaError_t bwd_tc_r_side(const bf16* qt0_16, const bf16* k, const bf16* v, const bf16* dkt16,
                          const bf16* dy16, const float* dhs, float* dqt0_part, bf16* dk,
                          bf16* dv, const Problem& pb, int* status, cudaStream_t stream,
                          int* launches) {
  if (!bwd_tc_r_side_supports(pb)) return cudaErrorInvalidValue;
  return pb.d == 128 ? launch_rbw<128>(qt0_16, k, v, dkt16, dy16, dhs, dqt0_part, dk, dv, pb,
                                       status, stream, launches)
                     : launch_rbw<64>(qt0_16, k, v, dkt16, dy16, dhs, dqt0_part, dk, dv, pb,
                                      status, stream, launches);
}

}  // namespace monarch
