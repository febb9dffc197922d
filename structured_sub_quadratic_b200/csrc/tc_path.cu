// tcgen05 tensor-core path for bf16 inputs.
//
// The final L-update fused with the output (the dominant FLOPs) runs on the
// 5th-generation tensor cores: for every (head g, position i, row group p)
// it is an attention of the |p| queries q_(l,i) against the b1*c2 keys
// Kt_{k,p,q,i} with a per-key bias Hs and values Y
// (MonarchAttention OpenReview discussion: the intermediate steps are
// FlashAttention-like calls; MonarchRT summary, "Method" (3): the N x N
// matrix is never formed):
//
//   S = q Kt^T / sqrt(d) + Hs          128 x NK tile, accumulated in TMEM
//   L = softmax over (k, q) of S        online, one TMEM lane (row) per thread
//   O = L Y                             128 x d, accumulated in TMEM
//
// Operands are staged by TMA with 128-byte swizzle: Q through a 3-D tensor
// map (rows l of one position i are b2*d elements apart), Kt and Y through
// 2-D maps over the position-major workspace.  One thread issues the
// tcgen05.mma instructions; four warps own the 128 rows for the softmax.
// The running max is only raised when a tile's max exceeds it by more than
// 2^8 (exact result, fewer rescales of the TMEM accumulator).
//
// Step one (aggregated queries under the uniform L, R-update) also runs on
// the tensor cores; later steps of T >= 2 run on the SIMT kernels.
#include "tc_path.cuh"

#include <cudaTypedefs.h>

#include <mutex>

#include "simt_kernels.cuh"
#include "tc_ptx.cuh"
#include "timing.cuh"

namespace monarch {

namespace {

using namespace tc;

constexpr int kRows = 128;  // query rows per CTA = UMMA M = TMEM lanes
constexpr int kThreadsKO = 128;
constexpr float kLog2e = 1.4426950408889634f;

template <int D, int NK>
struct KOLayout {
  static constexpr int kQBytes = D / 64 * kRows * 128;
  static constexpr int kKtBytes = D / 64 * NK * 128;
  static constexpr int kStageBytes = 2 * kKtBytes;  // Kt then Y
  static constexpr int kStages = 2;
  static constexpr int kPBytes = NK / 64 * kRows * 128;
  static constexpr int kStageOff = kQBytes;
  static constexpr int kPOff = kStageOff + kStages * kStageBytes;
  static constexpr int kBiasOff = kPOff + kPBytes;             // float [2][NK]
  static constexpr int kBarOff = kBiasOff + 2 * NK * 4;         // 8 x u64
  static constexpr int kBytes = kBarOff + 8 * 8;
  static constexpr int kAlloc = kBytes;  // the dynamic buffer is declared 1024-B aligned
  static constexpr uint32_t kTmemCols = (D + NK <= 128) ? 128u : (D + NK <= 256 ? 256u : 512u);
  static_assert(D % 64 == 0 && NK % 64 == 0, "tile sizes");
};

struct KOArgs {
  const float* hs;  // [G][b2][c1][nk]
  bf16* out;        // (G, N, d)
  int b1, b2, c1, nk, row_tiles;
  float sc_log2;    // log2(e) / sqrt(d)
  int* status;
};

// Thread-0 bookkeeping of asynchronous work in flight, so that an aborted
// CTA can drain it (bounded) before releasing TMEM.
struct InFlight {
  int kv_issued = 0, kv_waited = 0;
  int s_issued = 0, pv_issued = 0;
  bool q_waited = false;
};

__device__ __forceinline__ void drain(uint64_t* bar, uint32_t parity) {
  const unsigned long long t0 = global_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_ns() - t0 > kWaitLimitNs) break;
  }
}

template <int D, int NK>
__global__ void __launch_bounds__(kThreadsKO)
    ko_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kt,
              const __grid_constant__ CUtensorMap tm_y, KOArgs a) {
  using L = KOLayout<D, NK>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5;
  if (smem_u32(smem) & 1023u) {  // swizzled tiles need 1024-B alignment: report, never fault
    if (tid == 0) atomicExch(a.status, 2);
    return;
  }

  int bid = blockIdx.x;
  const int rt = bid % a.row_tiles;
  bid /= a.row_tiles;
  const int p = bid % a.c1;
  bid /= a.c1;
  const int i = bid % a.b2;
  const int g = bid / a.b2;
  const int l0 = group_start(a.b1, a.c1, p), l1 = group_start(a.b1, a.c1, p + 1);
  const int row0 = l0 + rt * kRows;
  if (row0 >= l1) return;  // whole CTA past the group: uniform, before any sync
  const int nrows = min(kRows, l1 - row0);
  const long key_row0 = ((long)(g * a.b2 + i) * a.c1 + p) * a.nk;
  const int nt = (a.nk + NK - 1) / NK;

  uint8_t* sQ = smem;
  uint8_t* sP = smem + L::kPOff;
  float* sBias = reinterpret_cast<float*>(smem + L::kBiasOff);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* q_full = bars + 0;
  uint64_t* kv_full = bars + 1;  // two stages
  uint64_t* s_full = bars + 3;
  uint64_t* pv_done = bars + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 6);
  auto sKt = [&](int st) { return smem + L::kStageOff + st * L::kStageBytes; };
  auto sY = [&](int st) { return smem + L::kStageOff + st * L::kStageBytes + L::kKtBytes; };

  if (tid == 0) {
    mbar_init(q_full, 1);
    mbar_init(kv_full, 1);
    mbar_init(kv_full + 1, 1);
    mbar_init(s_full, 1);
    mbar_init(pv_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (tid < NK) sBias[tid] = tid < a.nk ? a.hs[key_row0 + tid] * kLog2e : 0.f;
  if (warp == 0) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tmem_o = tmem;      // columns [0, D): output accumulator
  const uint32_t tmem_s = tmem + D;  // columns [D, D + NK): logits tile
  const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;

  InFlight fl;
  auto issue_kv = [&](int j) {
    const int st = j & 1;
    mbar_arrive_expect_tx(kv_full + st, L::kStageBytes);
    const int y = static_cast<int>(key_row0 + (long)j * NK);
#pragma unroll
    for (int c = 0; c < D / 64; ++c) {
      tma_load_2d(sKt(st) + c * NK * 128, &tm_kt, kv_full + st, c * 64, y);
      tma_load_2d(sY(st) + c * NK * 128, &tm_y, kv_full + st, c * 64, y);
    }
    ++fl.kv_issued;
  };
  if (tid == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_kt);
    tma_prefetch_desc(&tm_y);
    mbar_arrive_expect_tx(q_full, L::kQBytes);
#pragma unroll
    for (int c = 0; c < D / 64; ++c)
      tma_load_3d(sQ + c * kRows * 128, &tm_q, q_full, c * 64, i, g * a.b1 + row0);
    issue_kv(0);
    if (nt > 1) issue_kv(1);
  }

  const uint32_t idesc_s = idesc_bf16(kRows, NK, false);
  const uint32_t idesc_o = idesc_bf16(kRows, D, true);
  const int row = tid;
  float m_run = -INFINITY, l_run = 0.f;

  for (int j = 0; j < nt; ++j) {
    const int st = j & 1;
    // ---- S = Q Kt^T (one thread issues) ----
    if (tid == 0) {
      bool w = mbar_wait(kv_full + st, (j >> 1) & 1, abort_flag, a.status);
      if (w) ++fl.kv_waited;
      if (w && j == 0) {
        w = mbar_wait(q_full, 0, abort_flag, a.status);
        fl.q_waited = w;
      }
      if (w) {
        tc_fence_after();
        const uint32_t qb = smem_u32(sQ), kb = smem_u32(sKt(st));
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t ad = desc_kmajor(qb + (kk >> 2) * (kRows * 128) + (kk & 3) * 32);
          const uint64_t bd = desc_kmajor(kb + (kk >> 2) * (NK * 128) + (kk & 3) * 32);
          mma_bf16_ss(tmem_s, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
        }
        mma_commit(s_full);
        ++fl.s_issued;
      }
    }
    bool ok = mbar_wait(s_full, j & 1, abort_flag, a.status);
    ok = __all_sync(0xffffffffu, ok);

    // ---- softmax of this row's NK logits ----
    float sv[NK];
    float alpha = 1.f;
    bool resc = false;
    if (ok) {
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < NK / 32; ++c) {
        float t[32];
        tmem_ld32(tmem_s + lane_off + c * 32, t);
#pragma unroll
        for (int e = 0; e < 32; ++e) sv[c * 32 + e] = t[e];
      }
      tmem_wait_ld();
      const float* bias = sBias + st * NK;
      const int valid = a.nk - j * NK;
      float mt = -INFINITY;
#pragma unroll
      for (int c = 0; c < NK; ++c) {
        sv[c] = c < valid ? fmaf(sv[c], a.sc_log2, bias[c]) : -INFINITY;
        mt = fmaxf(mt, sv[c]);
      }
      if (mt > m_run + 8.f) {  // first tile, or the max grew by more than 2^8
        alpha = ex2(m_run - mt);
        resc = j > 0;
        m_run = mt;
      }
      float ls = 0.f;
#pragma unroll
      for (int c = 0; c < NK; ++c) {
        sv[c] = ex2(sv[c] - m_run);
        ls += sv[c];
      }
      l_run = l_run * alpha + ls;
    }
    // ---- previous P V done: P buffer free, O stable, its stage free ----
    if (ok && j > 0) ok = mbar_wait(pv_done, (j - 1) & 1, abort_flag, a.status);
    ok = __all_sync(0xffffffffu, ok);
    if (ok && tid == 0 && j >= 1 && j + 1 < nt) issue_kv(j + 1);
    if (ok && __any_sync(0xffffffffu, resc)) {
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        float t[32];
        tmem_ld32(tmem_o + lane_off + c * 32, t);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) t[e] *= alpha;
        tmem_st32(tmem_o + lane_off + c * 32, t);
      }
      tmem_wait_st();
    }
    if (ok) {
      // P row -> shared memory, K-major with 128-byte swizzle
#pragma unroll
      for (int u = 0; u < NK / 8; ++u) {
        uint4 pk;
        pk.x = pack_bf16x2(sv[8 * u + 0], sv[8 * u + 1]);
        pk.y = pack_bf16x2(sv[8 * u + 2], sv[8 * u + 3]);
        pk.z = pack_bf16x2(sv[8 * u + 4], sv[8 * u + 5]);
        pk.w = pack_bf16x2(sv[8 * u + 6], sv[8 * u + 7]);
        const int chunk = u >> 3, unit = u & 7;
        *reinterpret_cast<uint4*>(sP + chunk * (kRows * 128) + row * 128 +
                                  ((unit ^ (row & 7)) << 4)) = pk;
      }
      fence_proxy_async_smem();
    }
    if (tid < NK && j + 1 < nt) {
      const int col = (j + 1) * NK + tid;
      sBias[((j + 1) & 1) * NK + tid] = col < a.nk ? a.hs[key_row0 + col] * kLog2e : 0.f;
    }
    tc_fence_before();
    __syncthreads();
    if (*abort_flag) break;  // read after the barrier: uniform across the CTA
    // ---- O += P Y ----
    if (tid == 0) {
      tc_fence_after();
      const uint32_t pb = smem_u32(sP), yb = smem_u32(sY(st));
#pragma unroll
      for (int kk = 0; kk < NK / 16; ++kk) {
        const uint64_t ad = desc_kmajor(pb + (kk >> 2) * (kRows * 128) + (kk & 3) * 32);
        const uint64_t bd = desc_mnmajor(yb + kk * 16 * 128, NK * 128);
        mma_bf16_ss(tmem_o, ad, bd, idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
      }
      mma_commit(pv_done);
      ++fl.pv_issued;
    }
  }

  // ---- epilogue: O / l -> global ----
  bool ok = !*abort_flag && mbar_wait(pv_done, (nt - 1) & 1, abort_flag, a.status);
  ok = __all_sync(0xffffffffu, ok);
  if (ok) {
    tc_fence_after();
    const float inv = 1.f / l_run;
    const bool valid = row < nrows;
    bf16* orow = a.out + (((long)g * a.b1 + row0 + row) * a.b2 + i) * D;
#pragma unroll 1
    for (int c = 0; c < D / 32; ++c) {
      float t[32];
      tmem_ld32(tmem_o + lane_off + c * 32, t);
      tmem_wait_ld();
      if (valid) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          uint4 pk;
          pk.x = pack_bf16x2(t[8 * u + 0] * inv, t[8 * u + 1] * inv);
          pk.y = pack_bf16x2(t[8 * u + 2] * inv, t[8 * u + 3] * inv);
          pk.z = pack_bf16x2(t[8 * u + 4] * inv, t[8 * u + 5] * inv);
          pk.w = pack_bf16x2(t[8 * u + 6] * inv, t[8 * u + 7] * inv);
          *reinterpret_cast<uint4*>(orow + c * 32 + 8 * u) = pk;
        }
      }
    }
  }
  // ---- aborted: drain what is still in flight (bounded) before freeing TMEM ----
  if (tid == 0 && *abort_flag) {
    if (!fl.q_waited) drain(q_full, 0);
    for (int j = fl.kv_waited; j < fl.kv_issued; ++j) drain(kv_full + (j & 1), (j >> 1) & 1);
    if (fl.s_issued > 0) drain(s_full, (fl.s_issued - 1) & 1);
    if (fl.pv_issued > 0) drain(pv_done, (fl.pv_issued - 1) & 1);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Step-one aggregated queries under the uniform initial L (bf16):
// Qt0[g][p][i][:] = mean_{l in p} q_(l,i).  One block per (g, p, i); 16-byte
// column chunks x row lanes, reduced through shared memory.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256)
    init_qt_bf16_kernel(const bf16* __restrict__ q, bf16* __restrict__ qt0, int b1, int b2,
                        int c1) {
  constexpr int CH = D / 8;
  constexpr int LANES = 256 / CH;
  __shared__ float red[LANES][D];
  int bid = blockIdx.x;
  const int i = bid % b2;
  bid /= b2;
  const int p = bid % c1;
  const long g = bid / c1;
  const int l0 = group_start(b1, c1, p), l1 = group_start(b1, c1, p + 1);
  const int ch = threadIdx.x % CH, lane = threadIdx.x / CH;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  for (int l = l0 + lane; l < l1; l += LANES) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(q + ((g * b1 + l) * b2 + i) * D) + ch);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      acc[2 * e] += __uint_as_float(w[e] << 16);
      acc[2 * e + 1] += __uint_as_float(w[e] & 0xffff0000u);
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) red[lane][ch * 8 + e] = acc[e];
  __syncthreads();
  if (threadIdx.x < D) {
    float sum = 0.f;
#pragma unroll 4
    for (int ln = 0; ln < LANES; ++ln) sum += red[ln][threadIdx.x];
    qt0[((g * c1 + p) * b2 + i) * D + threadIdx.x] = __float2bfloat16_rn(sum / (float)(l1 - l0));
  }
}

// ---------------------------------------------------------------------------
// R-update of step one on the tensor cores.  One CTA per (g, k, p): the b2
// aggregated queries Qt0_{p,i} (rows, <= 128) against the b2 keys of chunk k:
//   S = Qt0 K_k^T / sqrt(d)                      128 x bk in TMEM
//   per column group q: R = softmax_{j in q}(S), Hs = entropy of R
//   [Kt | Y] = R [K_k | V_k]                      one N = 2d MMA chain
// The same K tile is the K-major B operand of the first product and the
// MN-major B operand of the second; [K | V] sit side by side in shared
// memory so their four 64-column blocks are one MN-major operand.  The
// output accumulator reuses the TMEM columns of S (S is in registers by
// then), so a CTA holds 2d columns.
// ---------------------------------------------------------------------------
struct KRArgs {
  bf16* kt;   // [G][b2][c1][b1][c2][d]
  bf16* y;
  float* hs;  // [G][b2][c1][b1][c2]
  int b1, b2, c1, c2, bk, write_y;
  float sc_log2;
  int* status;
};

template <int D>
struct KRLayout {
  int kv_box, q_off, k_off, v_off, p_off, bar_off, bytes;
  __host__ __device__ explicit KRLayout(int bk) {
    kv_box = bk * 128;
    q_off = 0;
    k_off = D / 64 * kRows * 128;
    v_off = k_off + D / 64 * kv_box;
    p_off = v_off + D / 64 * kv_box;
    bar_off = p_off + ((bk + 63) / 64) * kRows * 128;
    bytes = bar_off + 64;
  }
  static constexpr uint32_t kTmemCols = 2 * D;  // >= bk for bk <= 128
};

template <int D, int BKMAX>
__global__ void __launch_bounds__(128)
    kr_kernel(const __grid_constant__ CUtensorMap tm_qt, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, KRArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5;
  if (smem_u32(smem) & 1023u) {
    if (tid == 0) atomicExch(a.status, 2);
    return;
  }
  const KRLayout<D> L(a.bk);
  int bid = blockIdx.x;
  const int p = bid % a.c1;
  bid /= a.c1;
  const int k = bid % a.b1;
  const int g = bid / a.b1;
  const int bk = a.bk;

  uint8_t* sQ = smem + L.q_off;
  uint8_t* sK = smem + L.k_off;
  uint8_t* sV = smem + L.v_off;
  uint8_t* sP = smem + L.p_off;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bar_off);
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
    tmem_alloc(tmem_slot, KRLayout<D>::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;

  bool load_waited = false;
  int mma_issued = 0;  // commits outstanding on s_full / o_full, for the abort drain
  if (tid == 0) {
    tma_prefetch_desc(&tm_qt);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    mbar_arrive_expect_tx(load_full, D / 64 * (kRows * 128 + 2 * L.kv_box));
    const int qrow = (g * a.c1 + p) * a.b2;
    const int krow = (g * a.b1 + k) * a.b2;
#pragma unroll
    for (int c = 0; c < D / 64; ++c) {
      tma_load_2d(sQ + c * kRows * 128, &tm_qt, load_full, c * 64, qrow);
      tma_load_2d(sK + c * L.kv_box, &tm_k, load_full, c * 64, krow);
      tma_load_2d(sV + c * L.kv_box, &tm_v, load_full, c * 64, krow);
    }
    load_waited = mbar_wait(load_full, 0, abort_flag, a.status);
    if (load_waited) {
      tc_fence_after();
      const uint32_t qb = smem_u32(sQ), kb = smem_u32(sK);
      const uint32_t idesc = idesc_bf16(kRows, bk, false);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint64_t ad = desc_kmajor(qb + (kk >> 2) * (kRows * 128) + (kk & 3) * 32);
        const uint64_t bd = desc_kmajor(kb + (kk >> 2) * L.kv_box + (kk & 3) * 32);
        mma_bf16_ss(tmem, ad, bd, idesc, kk > 0 ? 1u : 0u);
      }
      mma_commit(s_full);
      mma_issued = 1;
    }
  }
  bool ok = mbar_wait(s_full, 0, abort_flag, a.status);
  ok = __all_sync(0xffffffffu, ok);
  float sv[BKMAX];
  if (ok) {
    tc_fence_after();
#pragma unroll
    for (int c = 0; c < BKMAX / 32; ++c) {
      float t[32];
      tmem_ld32(tmem + lane_off + c * 32, t);
#pragma unroll
      for (int e = 0; e < 32; ++e) sv[c * 32 + e] = t[e] * a.sc_log2;
    }
    tmem_wait_ld();
  }
  const int r = tid;  // row = position i
  const bool row_valid = r < a.b2;
  for (int q = 0; q < a.c2; ++q) {
    const int j0 = group_start(a.b2, a.c2, q), j1 = group_start(a.b2, a.c2, q + 1);
    float m2 = -INFINITY;
#pragma unroll
    for (int j = 0; j < BKMAX; ++j)
      if (j >= j0 && j < j1) m2 = fmaxf(m2, sv[j]);
    float z = 0.f, t2 = 0.f;
    if (ok) {
#pragma unroll
      for (int u = 0; u < BKMAX / 8; ++u) {
        if (u * 8 >= bk) break;
        float e8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int j = u * 8 + e;
          const float x = (j >= j0 && j < j1) ? ex2(sv[j] - m2) : 0.f;
          e8[e] = __bfloat162float(__float2bfloat16_rn(x));
          z += e8[e];
          t2 += (j >= j0 && j < j1) ? e8[e] * (sv[j] - m2) : 0.f;
        }
        uint4 pk;
        pk.x = pack_bf16x2(e8[0], e8[1]);
        pk.y = pack_bf16x2(e8[2], e8[3]);
        pk.z = pack_bf16x2(e8[4], e8[5]);
        pk.w = pack_bf16x2(e8[6], e8[7]);
        const int chunk = u >> 3, unit = u & 7;
        *reinterpret_cast<uint4*>(sP + chunk * (kRows * 128) + r * 128 +
                                  ((unit ^ (r & 7)) << 4)) = pk;
      }
      fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    if (*abort_flag) break;
    if (tid == 0) {
      tc_fence_after();
      const uint32_t pb = smem_u32(sP), kb = smem_u32(sK);
      const uint32_t idesc = idesc_bf16(kRows, 2 * D, true);
      for (int kk = 0; kk < bk / 16; ++kk) {
        const uint64_t ad = desc_kmajor(pb + (kk >> 2) * (kRows * 128) + (kk & 3) * 32);
        const uint64_t bd = desc_mnmajor(kb + kk * 16 * 128, L.kv_box);
        mma_bf16_ss(tmem, ad, bd, idesc, kk > 0 ? 1u : 0u);
      }
      mma_commit(o_full);
      ++mma_issued;
    }
    ok = mbar_wait(o_full, q & 1, abort_flag, a.status);
    ok = __all_sync(0xffffffffu, ok);
    if (ok) {
      tc_fence_after();
      const float inv = 1.f / z;
      const long orow = ((((long)g * a.b2 + r) * a.c1 + p) * a.b1 + k) * a.c2 + q;
#pragma unroll 1
      for (int half = 0; half < (a.write_y ? 2 : 1); ++half) {
        bf16* dst = (half == 0 ? a.kt : a.y) + orow * D;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          float t[32];
          tmem_ld32(tmem + lane_off + half * D + c * 32, t);
          tmem_wait_ld();
          if (row_valid) {
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              uint4 pk;
              pk.x = pack_bf16x2(t[8 * u + 0] * inv, t[8 * u + 1] * inv);
              pk.y = pack_bf16x2(t[8 * u + 2] * inv, t[8 * u + 3] * inv);
              pk.z = pack_bf16x2(t[8 * u + 4] * inv, t[8 * u + 5] * inv);
              pk.w = pack_bf16x2(t[8 * u + 6] * inv, t[8 * u + 7] * inv);
              *reinterpret_cast<uint4*>(dst + c * 32 + 8 * u) = pk;
            }
          }
        }
      }
      // entropy of the R row: ln z - sum e (s - m) / z, with s - m in log2 units
      if (row_valid) a.hs[orow] = logf(z) - t2 * 0.69314718055994531f * inv;
    }
    tc_fence_before();
    __syncthreads();
    if (*abort_flag) break;
  }
  if (tid == 0 && *abort_flag) {
    if (!load_waited) drain(load_full, 0);
    if (mma_issued >= 1) drain(s_full, 0);
    if (mma_issued >= 2) drain(o_full, (mma_issued - 2) & 1);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, KRLayout<D>::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// bf16 tensor map with 128-byte swizzle; dims/strides innermost first,
// strides in bytes for dims 1.. .
bool make_map(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims,
              const cuuint64_t* strides, const cuuint32_t* box) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int NK>
cudaError_t launch_ko(const bf16* q, const bf16* kt, const bf16* y, const float* hs, bf16* out,
                      const Problem& pb, int* status, cudaStream_t stream, int* launches) {
  using L = KOLayout<D, NK>;
  static std::once_flag attr_once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(attr_once, [] {
    attr_err = cudaFuncSetAttribute(ko_kernel<D, NK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    L::kAlloc);
  });
  if (attr_err != cudaSuccess) return attr_err;
  const int nk = pb.b1 * pb.c2;
  const long key_rows = (long)pb.G * pb.b2 * pb.c1 * nk;
  CUtensorMap tq, tk, tyv;
  {
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)pb.b2, (cuuint64_t)pb.G * pb.b1};
    const cuuint64_t str[2] = {(cuuint64_t)D * 2, (cuuint64_t)pb.b2 * D * 2};
    const cuuint32_t box[3] = {64, 1, kRows};
    if (!make_map(&tq, q, 3, dims, str, box)) return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)key_rows};
    const cuuint64_t str[1] = {(cuuint64_t)D * 2};
    const cuuint32_t box[2] = {64, NK};
    if (!make_map(&tk, kt, 2, dims, str, box)) return cudaErrorInvalidValue;
    if (!make_map(&tyv, y, 2, dims, str, box)) return cudaErrorInvalidValue;
  }
  const int gmax = (pb.b1 + pb.c1 - 1) / pb.c1;
  KOArgs a;
  a.hs = hs;
  a.out = out;
  a.b1 = pb.b1;
  a.b2 = pb.b2;
  a.c1 = pb.c1;
  a.nk = nk;
  a.row_tiles = (gmax + kRows - 1) / kRows;
  a.sc_log2 = kLog2e * pb.sc;
  a.status = status;
  const long blocks = (long)pb.G * pb.b2 * pb.c1 * a.row_tiles;
  return timed_launch("tc_l_output", stream, launches, [&] {
    ko_kernel<D, NK><<<(unsigned)blocks, kThreadsKO, L::kAlloc, stream>>>(tq, tk, tyv, a);
  });
}

template <int D, int BKMAX>
cudaError_t launch_kr(const bf16* qt0, const bf16* k, const bf16* v, bf16* kt, bf16* y, float* hs,
                      const Problem& pb, int bk, int* status, cudaStream_t stream,
                      int* launches) {
  const KRLayout<D> L(bk);
  static std::once_flag attr_once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(attr_once, [] {
    attr_err = cudaFuncSetAttribute(kr_kernel<D, BKMAX>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    KRLayout<D>(BKMAX).bytes);
  });
  if (attr_err != cudaSuccess) return attr_err;
  CUtensorMap tq, tk, tv;
  {
    const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)pb.G * pb.c1 * pb.b2};
    const cuuint64_t str[1] = {(cuuint64_t)D * 2};
    const cuuint32_t box[2] = {64, kRows};
    if (!make_map(&tq, qt0, 2, dims, str, box)) return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)pb.G * pb.b1 * pb.b2};
    const cuuint64_t str[1] = {(cuuint64_t)D * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)bk};
    if (!make_map(&tk, k, 2, dims, str, box)) return cudaErrorInvalidValue;
    if (!make_map(&tv, v, 2, dims, str, box)) return cudaErrorInvalidValue;
  }
  KRArgs a;
  a.kt = kt;
  a.y = y;
  a.hs = hs;
  a.b1 = pb.b1;
  a.b2 = pb.b2;
  a.c1 = pb.c1;
  a.c2 = pb.c2;
  a.bk = bk;
  a.write_y = pb.T == 1 ? 1 : 0;
  a.sc_log2 = kLog2e * pb.sc;
  a.status = status;
  const long blocks = (long)pb.G * pb.b1 * pb.c1;
  return timed_launch("tc_r_update", stream, launches, [&] {
    kr_kernel<D, BKMAX><<<(unsigned)blocks, 128, L.bytes, stream>>>(tq, tk, tv, a);
  });
}

// Step one: aggregated queries under the uniform L, then the R-update.
template <int D>
cudaError_t launch_r_step1(const bf16* q, const bf16* k, const bf16* v, bf16* qt0, bf16* kt,
                           bf16* y, float* hs, const Problem& pb, int* status,
                           cudaStream_t stream, int* launches) {
  cudaError_t e = timed_launch("tc_init_qt", stream, launches, [&] {
    init_qt_bf16_kernel<D><<<(unsigned)((long)pb.G * pb.c1 * pb.b2), 256, 0, stream>>>(
        q, qt0, pb.b1, pb.b2, pb.c1);
  });
  if (e != cudaSuccess) return e;
  const int bk = (pb.b2 + 15) / 16 * 16;
  if (bk <= 64) return launch_kr<D, 64>(qt0, k, v, kt, y, hs, pb, bk, status, stream, launches);
  return launch_kr<D, 128>(qt0, k, v, kt, y, hs, pb, bk, status, stream, launches);
}

constexpr size_t kAlign = 256;
size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// Workspace: the SIMT pieces with bf16 Kt/Y (position-major, the layout the
// tensor-core kernel reads through its 2-D tensor maps).
SimtWorkspace carve(const Problem& pb, char* base, size_t* total) {
  const SimtWorkspaceSizes s = simt_workspace_sizes(pb);
  const size_t bytes[7] = {s.qt0 * 4, s.qt * 4, s.kt * 2, s.y * 2, s.hs * 4, s.lse * 4, s.ybar * 4};
  void* ptr[7];
  size_t off = 0;
  for (int t = 0; t < 7; ++t) {
    ptr[t] = (base && bytes[t]) ? static_cast<void*>(base + off) : nullptr;
    off += align_up(bytes[t]);
  }
  if (total) *total = off;
  SimtWorkspace ws;
  ws.qt0 = static_cast<float*>(ptr[0]);
  ws.qt = static_cast<float*>(ptr[1]);
  ws.kt = ptr[2];
  ws.y = ptr[3];
  ws.hs = static_cast<float*>(ptr[4]);
  ws.lse = static_cast<float*>(ptr[5]);
  ws.ybar = static_cast<float*>(ptr[6]);
  return ws;
}

}  // namespace

bool tc_supports(const Problem& pb) {
  if (pb.d != 64 && pb.d != 128) return false;
  if (pb.T < 1 || pb.b2 > 128) return false;  // R-side tile: b2 keys <= 128 rows
  const long key_rows = (long)pb.G * pb.b2 * pb.c1 * pb.b1 * pb.c2;
  if (key_rows + 256 >= (1L << 31) || (long)pb.G * pb.b1 >= (1L << 31)) return false;
  return encode_fn() != nullptr;
}

size_t tc_workspace_bytes(const Problem& pb) {
  size_t total = 0;
  carve(pb, nullptr, &total);
  return total;
}

cudaError_t tc_forward(const bf16* q, const bf16* k, const bf16* v, bf16* out, const Problem& pb,
                       char* ws_base, int* status, cudaStream_t stream, int* launches) {
  const SimtWorkspace ws = carve(pb, ws_base, nullptr);
  bf16* kt = static_cast<bf16*>(ws.kt);
  bf16* y = static_cast<bf16*>(ws.y);
  bf16* qt0 = reinterpret_cast<bf16*>(ws.qt0);
  cudaError_t e = pb.d == 128 ? launch_r_step1<128>(q, k, v, qt0, kt, y, ws.hs, pb, status, stream,
                                                    launches)
                              : launch_r_step1<64>(q, k, v, qt0, kt, y, ws.hs, pb, status, stream,
                                                   launches);
  if (e != cudaSuccess) return e;
  const QtStrides s1 = {(long)pb.b1 * pb.c1 * pb.c2 * pb.b2 * pb.d,
                        (long)pb.c1 * pb.c2 * pb.b2 * pb.d, (long)pb.c2 * pb.b2 * pb.d,
                        (long)pb.b2 * pb.d, (long)pb.d};
  for (int t = 2; t <= pb.T; ++t) {
    e = simt_l_update<bf16, bf16>(q, kt, ws.hs, ws.lse, ws.qt, pb, stream, launches);
    if (e != cudaSuccess) return e;
    e = simt_r_update<bf16, bf16>(k, v, ws.qt, s1, kt, y, ws.hs, pb, t == pb.T, stream, launches);
    if (e != cudaSuccess) return e;
  }
  if (pb.d == 128) return launch_ko<128, 64>(q, kt, y, ws.hs, out, pb, status, stream, launches);
  return launch_ko<64, 64>(q, kt, y, ws.hs, out, pb, status, stream, launches);
}

}  // namespace monarch
