// tcgen05 tensor-core path for bf16 inputs.
//
// The final L-update fused with the output (the dominant FLOPs) runs on the
// 5th-generation tensor cores: for every (head g, position i, row group p)
// it is an attention of the |p| queries q_(l,i) against the b1*c2 keys
// Kt_{k,p,q,i} with a per-key bias Hs and values Y
// (MonarchAttention OpenReview discussion, author response on the kernels:
// each intermediate step is a fused attention-style call; MonarchRT
// summary, "Method" (3): the N x N matrix is never formed):
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
// the tensor cores, and so do the later steps of T >= 2 (non-final L-update
// with the aggregation L^T Q, R-update from per-sub-item queries).  Groups
// too small for a 128-row tile (a few keys or rows) take the CUDA-core
// kernels of small_dim.cu instead.
#include "tc_path.cuh"

#include <cudaTypedefs.h>

#include <mutex>
#include <utility>

#include "launch.cuh"
#include "simt_kernels.cuh"
#include "small_dim.cuh"
#include "tc_ptx.cuh"
#include "timing.cuh"

namespace monarch {

namespace {

using namespace tc;

constexpr int kRows = 128;  // query rows per CTA = UMMA M = TMEM lanes
constexpr float kLog2e = 1.4426950408889634f;
// Lazy rescale threshold of the output kernel: 8 in log2 units (a factor 2^8).
constexpr float kRescaleNat = 8.f * 0.69314718055994531f;

// Box coordinates (y, z) in the 3-D tensor maps of q (rows row0.. of
// position i) and of k, v (keys j0.. of chunk k), for Monarch token order
// (tr = 0) or its transpose (tr = 1); make_q_slab_map and make_kv_map build
// the maps.
__device__ __forceinline__ int2 q_slab_yz(int tr, int g, int b1, int b2, int i, int row0) {
  return tr ? make_int2(row0, g * b2 + i) : make_int2(i, g * b1 + row0);
}

__device__ __forceinline__ int2 kv_yz(int tr, int g, int b1, int b2, int k, int j0) {
  return tr ? make_int2(k, g * b2 + j0) : make_int2(j0, g * b1 + k);
}

template <int D, int NK>
struct KOLayout {
  static constexpr int kQBytes = D / 64 * kRows * 128;
  static constexpr int kTileBytes = D / 64 * NK * 128;  // one Kt or Y tile
  static constexpr int kPBytes = NK / 64 * kRows * 128;
  static constexpr int kKtOff = kQBytes;                 // Kt ring, 2 slots
  static constexpr int kYOff = kKtOff + 2 * kTileBytes;   // Y ring, 2 slots
  static constexpr int kPOff = kYOff + 2 * kTileBytes;
  static constexpr int kBiasOff = kPOff + kPBytes;        // float [2][NK]
  static constexpr int kBarOff = kBiasOff + 2 * NK * 4;
  static constexpr int kBytes = kBarOff + 24 * 8;
  // At most two CTAs per SM (their TMEM use is 2 x 256 columns).
  static constexpr int kAlloc = kBytes > 100 * 1024 ? kBytes : 100 * 1024;
  static constexpr uint32_t kTmemCols = 256;  // O: D columns, S: two buffers of NK
  static_assert(D % 64 == 0 && NK % 64 == 0 && D + 2 * NK <= 256, "tile sizes");
};

struct KOArgs {
  const float* hs;  // [G][b2][c1][nk]
  bf16* out;        // (G, N, d)
  int b1, b2, c1, nk, row_tiles, n_items;
  float sc;         // 1 / sqrt(d)
  int* status;
  int tr;           // token order (see Problem)
};

// First output row of a tile (row0 of position i of head g) and the stride
// between its rows, in elements.
__device__ __forceinline__ bf16* out_tile(const KOArgs& a, int g, int i, int row0, int d) {
  return a.out + (a.tr ? ((long)g * a.b2 + i) * a.b1 + row0 : ((long)g * a.b1 + row0) * a.b2 + i) *
                     d;
}

__device__ __forceinline__ long out_stride(const KOArgs& a, int d) {
  return a.tr ? (long)d : (long)a.b2 * d;
}

__device__ __forceinline__ void drain(uint64_t* bar, uint32_t parity) {
  const unsigned long long t0 = global_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_ns() - t0 > kWaitLimitNs) break;
  }
}

// Work item = one 128-row query tile of one (g, i, p).  Returns false for
// tiles past the end of the row group (possible when groups differ in size).
struct KOItem {
  int g, i, p, row0, nrows, nt;
  long key_row0;
};

template <int NK>
__device__ __forceinline__ bool ko_decode(const KOArgs& a, int item, KOItem& it) {
  int bid = item;
  const int rt = bid % a.row_tiles;
  bid /= a.row_tiles;
  it.p = bid % a.c1;
  bid /= a.c1;
  it.i = bid % a.b2;
  it.g = bid / a.b2;
  const int l0 = group_start(a.b1, a.c1, it.p), l1 = group_start(a.b1, a.c1, it.p + 1);
  it.row0 = l0 + rt * kRows;
  if (it.row0 >= l1) return false;
  it.nrows = min(kRows, l1 - it.row0);
  it.key_row0 = ((long)(it.g * a.b2 + it.i) * a.c1 + it.p) * a.nk;
  it.nt = (a.nk + NK - 1) / NK;
  return true;
}

// Epilogue of the output kernels (four softmax warps, thread = tile row):
// O / l from TMEM to the rows' global memory.  TMEM loads run one 32-column
// unit ahead of the staging; each 64-column half is staged (swizzled) in
// sP, then 8 threads write one row's 128-byte half, so global stores are
// whole sectors.  o_empty is arrived on as soon as the last TMEM load of O
// has landed, so the next item's P Y may start while the rows go out.
template <int D>
__device__ __forceinline__ void ko_epilogue(uint32_t tmem_o, uint32_t lane_off, int row, float inv,
                                            uint8_t* sP, bf16* out_rows, long row_stride,
                                            int nrows, uint64_t* o_empty) {
  const int srow = threadIdx.x - 64;  // 0..127 over the four softmax warps
  float rs[2][32];
  tmem_ld32(tmem_o + lane_off, rs[0]);
#pragma unroll
  for (int u = 0; u < D / 32; ++u) {
    const int h = u >> 1, c = u & 1;
    tmem_wait_ld();  // unit u is in registers
    if (u == D / 32 - 1) {  // O fully read: the next P Y may overwrite it
      tc_fence_before();
      mbar_arrive(o_empty);
    } else {
      tmem_ld32(tmem_o + lane_off + (u + 1) * 32, rs[(u + 1) & 1]);
    }
#pragma unroll
    for (int uu = 0; uu < 4; ++uu) {
      const float* t = rs[u & 1] + 8 * uu;
      uint4 pk;
      pk.x = pack_bf16x2(t[0] * inv, t[1] * inv);
      pk.y = pack_bf16x2(t[2] * inv, t[3] * inv);
      pk.z = pack_bf16x2(t[4] * inv, t[5] * inv);
      pk.w = pack_bf16x2(t[6] * inv, t[7] * inv);
      const int unit = c * 4 + uu;
      *reinterpret_cast<uint4*>(sP + row * 128 + ((unit ^ (row & 7)) << 4)) = pk;
    }
    if (c == 1) {
      named_barrier(1, 128);
#pragma unroll
      for (int pass = 0; pass < kRows / 16; ++pass) {
        const int r = pass * 16 + (srow >> 3), unit = srow & 7;
        if (r < nrows) {
          const uint4 v4 = *reinterpret_cast<const uint4*>(sP + r * 128 + ((unit ^ (r & 7)) << 4));
          *reinterpret_cast<uint4*>(out_rows + r * row_stride + h * 64 + unit * 8) = v4;
        }
      }
      named_barrier(1, 128);
    }
  }
}

// Persistent, warp-specialised L-update + output.  Warp 0 loads Q, Kt, Y
// (TMA) and the entropy bias (plain loads), warp 1 issues the tcgen05.mma
// instructions from one thread, warps 2-5 own the 128 rows (TMEM lanes) for
// the online softmax and the epilogue.  Kt and Y have
// separate two-slot rings: a Kt slot is recycled as soon as its S tile is
// computed, a Y slot once its P Y product is, so each load is issued about
// two tiles before it is needed.  mbarriers hand tiles between roles:
//   q_full/q_empty          Q tile (one per item)
//   kt_full/kt_empty        Kt ring          y_full/y_empty   Y ring
//   bias_full/bias_empty    bias ring        s_full[2]        S tile in TMEM buffer
//   p_full[2]               P of the tile written over its S (TMEM, bf16 pairs)
//   pv_done[2]              O += P Y of the tile complete (its S/P buffer free,
//                           O stable)
// P never leaves the tensor memory: the softmax overwrites its S tile with P
// and the P Y product reads A from TMEM, so S and P are double-buffered.
//   o_empty                 epilogue has read O (next item may overwrite it)
// All counters run over the tiles T of every item this CTA processes.
template <int D, int NK>
__global__ void __launch_bounds__(192, 2)
    ko_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kt,
              const __grid_constant__ CUtensorMap tm_y, KOArgs a) {
  using L = KOLayout<D, NK>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (smem_u32(smem) & 1023u) {  // swizzled tiles need 1024-B alignment: report, never fault
    if (tid == 0) atomicExch(a.status, 2);
    return;
  }
  pdl_launch_dependents();
  uint8_t* sQ = smem;
  uint8_t* sP = smem + L::kPOff;
  float* sBias = reinterpret_cast<float*>(smem + L::kBiasOff);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* kt_full = bars + 2;      // [2]
  uint64_t* kt_empty = bars + 4;     // [2]
  uint64_t* y_full = bars + 6;       // [2]
  uint64_t* y_empty = bars + 8;      // [2]
  uint64_t* s_full = bars + 10;      // [2]
  uint64_t* pv_done = bars + 12;     // [2]
  uint64_t* bias_full = bars + 14;   // [2]
  uint64_t* bias_empty = bars + 16;  // [2]
  uint64_t* p_full = bars + 18;      // [2]
  uint64_t* o_empty = bars + 20;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 21);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 22);
  auto sKt = [&](int st) { return smem + L::kKtOff + st * L::kTileBytes; };
  auto sY = [&](int st) { return smem + L::kYOff + st * L::kTileBytes; };

  if (tid == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(kt_full + s, 1);
      mbar_init(kt_empty + s, 1);
      mbar_init(y_full + s, 1);
      mbar_init(y_empty + s, 1);
      mbar_init(s_full + s, 1);
      mbar_init(pv_done + s, 1);
      mbar_init(p_full + s, 128);
      mbar_init(bias_full + s, 32);
      mbar_init(bias_empty + s, 128);
    }
    mbar_init(o_empty, 128);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tmem_o = tmem;  // columns [0, D)
  auto tmem_s = [&](int sb) { return tmem + D + sb * NK; };

  auto first_item = [&](int item, KOItem& it) {
    for (; item < a.n_items; item += gridDim.x)
      if (ko_decode<NK>(a, item, it)) return item;
    return a.n_items;
  };
  if (warp == 0) {
    // ------------------- producer: Q, Kt + bias, Y (event-driven) -------------------
    // Two cursors walk the tiles: Kt (with the bias, and Q at an item's first
    // tile) and Y; each load is issued as soon as its slot is free.  Lane 0
    // probes the barriers and issues TMA; all lanes copy the bias.
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_kt);
      tma_prefetch_desc(&tm_y);
    }
    KOItem kit, yit;
    int k_item = first_item(blockIdx.x, kit), y_item = first_item(blockIdx.x, yit);
    int k_j = 0, k_n = 0, y_j = 0;
    long Tk = 0, Ty = 0;
    bool ok = true, waited = false;
    unsigned long long idle_since = global_ns();
    while ((k_item < a.n_items || y_item < a.n_items) && ok) {
      bool progressed = false;
      if (k_item < a.n_items) {
        const int st = (int)(Tk & 1);
        int ready = 0;
        if (lane == 0)
          ready = (k_j > 0 || k_n == 0 || mbar_test(q_empty, (k_n - 1) & 1)) &&
                  (Tk < 2 || (mbar_test(kt_empty + st, ((Tk >> 1) - 1) & 1) &&
                              mbar_test(bias_empty + st, ((Tk >> 1) - 1) & 1)));
        if (__shfl_sync(0xffffffffu, ready, 0)) {
          if (lane == 0 && k_j == 0) {
            const int2 qyz = q_slab_yz(a.tr, kit.g, a.b1, a.b2, kit.i, kit.row0);
            mbar_arrive_expect_tx(q_full, L::kQBytes);
#pragma unroll
            for (int c = 0; c < D / 64; ++c)
              tma_load_3d(sQ + c * kRows * 128, &tm_q, q_full, c * 64, qyz.x, qyz.y);
          }
          if (!waited) {  // Kt, Y and the bias come from the previous kernel
            pdl_wait();
            waited = true;
          }
          const int y = static_cast<int>(kit.key_row0 + (long)k_j * NK);
          if (lane == 0) {
            mbar_arrive_expect_tx(kt_full + st, L::kTileBytes);
#pragma unroll
            for (int c = 0; c < D / 64; ++c)
              tma_load_2d(sKt(st) + c * NK * 128, &tm_kt, kt_full + st, c * 64, y);
          }
          // the tile's entropy bias, copied asynchronously (columns past nk
          // are left stale; the softmax masks them)
          float* bias = sBias + st * NK;
          for (int e = lane; e < NK; e += 32) {
            const int col = k_j * NK + e;
            if (col < a.nk) cp_async_4(bias + e, a.hs + kit.key_row0 + col);
          }
          cp_async_arrive_noinc(bias_full + st);
          ++Tk;
          if (++k_j == kit.nt) {
            k_j = 0;
            ++k_n;
            k_item = first_item(k_item + gridDim.x, kit);
          }
          progressed = true;
        }
      }
      if (y_item < a.n_items && Ty < Tk) {
        const int st = (int)(Ty & 1);
        int ready = 0;
        if (lane == 0) ready = Ty < 2 || mbar_test(y_empty + st, ((Ty >> 1) - 1) & 1);
        if (__shfl_sync(0xffffffffu, ready, 0)) {
          if (lane == 0) {
            mbar_arrive_expect_tx(y_full + st, L::kTileBytes);
            const int y = static_cast<int>(yit.key_row0 + (long)y_j * NK);
#pragma unroll
            for (int c = 0; c < D / 64; ++c)
              tma_load_2d(sY(st) + c * NK * 128, &tm_y, y_full + st, c * 64, y);
          }
          ++Ty;
          if (++y_j == yit.nt) {
            y_j = 0;
            y_item = first_item(y_item + gridDim.x, yit);
          }
          progressed = true;
        }
      }
      if (progressed) {
        idle_since = global_ns();
      } else {
        __nanosleep(32);
        int bad = 0;
        if (lane == 0) {
          if (*abort_flag) {
            bad = 1;
          } else if (global_ns() - idle_since > kWaitLimitNs) {
            *abort_flag = 1;
            atomicExch(a.status, 1);
            bad = 1;
          }
        }
        ok = !__shfl_sync(0xffffffffu, bad, 0);
      }
    }
    if (lane == 0 && *abort_flag) {  // drain the loads this warp issued (bounded)
      if (k_n >= 1 || k_j > 0) drain(q_full, (k_j > 0 ? k_n : k_n - 1) & 1);
      for (long t = (Tk >= 2 ? Tk - 2 : 0); t < Tk; ++t) drain(kt_full + (t & 1), (t >> 1) & 1);
      for (long t = (Ty >= 2 ? Ty - 2 : 0); t < Ty; ++t) drain(y_full + (t & 1), (t >> 1) & 1);
    }
  } else if (warp == 1) {
    // -------------------------------- MMA ---------------------------------
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16(kRows, NK, false);
      const uint32_t idesc_o = idesc_bf16(kRows, D, true);
      long last_s = -1, last_pv = -1;
      bool ok = true;
      // Base descriptors, built once; each MMA adds a compile-time offset.
      const uint64_t dq = desc_kmajor(smem_u32(sQ));
      const uint64_t dkt0 = desc_kmajor(smem_u32(sKt(0))), dkt1 = desc_kmajor(smem_u32(sKt(1)));
      const uint64_t dy0 = desc_mnmajor(smem_u32(sY(0)), NK * 128),
                     dy1 = desc_mnmajor(smem_u32(sY(1)), NK * 128);
      // Event-driven issue over two cursors (next S tile, next P Y tile):
      // whichever has its inputs ready goes out first.
      KOItem sit, pit;
      int s_item = first_item(blockIdx.x, sit), p_item = first_item(blockIdx.x, pit);
      int s_j = 0, s_n = 0, p_j = 0, p_n = 0;
      long Ts = 0, Tp = 0;
      unsigned long long idle_since = global_ns();
      while (p_item < a.n_items && ok) {
        bool progressed = false;
        if (s_item < a.n_items) {
          const int st = (int)(Ts & 1);
          if ((s_j > 0 || mbar_test(q_full, s_n & 1)) && mbar_test(kt_full + st, (Ts >> 1) & 1) &&
              (Ts < 2 || mbar_test(pv_done + st, ((Ts >> 1) - 1) & 1))) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
              mma_bf16_ss(tmem_s(st), dq + (((kk >> 2) * (kRows * 128) + (kk & 3) * 32) >> 4),
                          (st ? dkt1 : dkt0) + (((kk >> 2) * (NK * 128) + (kk & 3) * 32) >> 4),
                          idesc_s,
                          kk > 0 ? 1u : 0u);
            mma_commit(s_full + st);
            mma_commit(kt_empty + st);
            last_s = Ts;
            ++Ts;
            if (++s_j == sit.nt) {
              mma_commit(q_empty);
              s_j = 0;
              ++s_n;
              s_item = first_item(s_item + gridDim.x, sit);
            }
            progressed = true;
          }
        }
        if (Tp < Ts) {
          const int st = (int)(Tp & 1);
          if (mbar_test(p_full + st, (Tp >> 1) & 1) && mbar_test(y_full + st, (Tp >> 1) & 1) &&
              (p_j > 0 || p_n == 0 || mbar_test(o_empty, (p_n - 1) & 1))) {
            tc_fence_after();
            // A = P from TMEM, 8 columns per 16 keys; a partial last tile
            // only over its valid keys (the rest of its P is not written)
            const int kk_n = min(NK / 16, (a.nk - p_j * NK + 15) / 16);
#pragma unroll
            for (int kk = 0; kk < NK / 16; ++kk)
              if (kk < kk_n)
                mma_bf16_ts(tmem_o, tmem_s(st) + kk * 8, (st ? dy1 : dy0) + ((kk * 16 * 128) >> 4),
                            idesc_o, (p_j > 0 || kk > 0) ? 1u : 0u);
            mma_commit(y_empty + st);
            mma_commit(pv_done + st);
            last_pv = Tp;
            ++Tp;
            if (++p_j == pit.nt) {
              p_j = 0;
              ++p_n;
              p_item = first_item(p_item + gridDim.x, pit);
            }
            progressed = true;
          }
        }
        if (progressed) {
          idle_since = global_ns();
        } else if ((__nanosleep(20), *abort_flag)) {
          ok = false;
        } else if (global_ns() - idle_since > kWaitLimitNs) {
          *abort_flag = 1;
          atomicExch(a.status, 1);
          ok = false;
        }
      }
      if (*abort_flag) {  // drain this thread's MMAs (bounded)
        if (last_s >= 0) drain(s_full + (last_s & 1), (last_s >> 1) & 1);
        if (last_pv >= 0) drain(pv_done + (last_pv & 1), (last_pv >> 1) & 1);
      }
    }
    __syncwarp();
  } else {
    // ------------------------- softmax + epilogue --------------------------
    const int quad = warp & 3;
    const int row = quad * 32 + lane;  // TMEM lane == tile row
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    long T = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < a.n_items && ok; item += gridDim.x) {
      KOItem it;
      if (!ko_decode<NK>(a, item, it)) continue;
      float m_run = -INFINITY, l_run = 0.f;
      for (int j = 0; j < it.nt; ++j, ++T) {
        const int sb = (int)(T & 1);
        ok = mbar_wait(s_full + sb, (T >> 1) & 1, abort_flag, a.status);
        if (ok) ok = mbar_wait(bias_full + sb, (T >> 1) & 1, abort_flag, a.status);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        float sv[NK];
        tc_fence_after();
        const float* bias = sBias + sb * NK;
        const int valid = a.nk - j * NK;
        // a last tile with at most NK/2 valid keys is handled at half width
        // (its other columns are neither read nor written)
        const bool half = valid <= NK / 2;
#pragma unroll
        for (int c = 0; c < NK / 32; ++c) {
          if (c == 0 || !half) {
            float t[32];
            tmem_ld32(tmem_s(sb) + lane_off + c * 32, t);
#pragma unroll
            for (int e = 0; e < 32; ++e) sv[c * 32 + e] = t[e];
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) sv[c * 32 + e] = -INFINITY;
          }
        }
        tmem_wait_ld();
        // logits sc q.Kt + Hs (natural units); 4 partial maxima / sums break
        // the serial chains
        float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        if (valid >= NK) {
          // packed pairs: the same roundings as the scalar forms, half the
          // instructions (the softmax warps share their schedulers)
          const float2 sc2 = make_float2(a.sc, a.sc);
#pragma unroll
          for (int c = 0; c < NK; c += 4) {
            const float4 b4 = *reinterpret_cast<const float4*>(bias + c);
            const float2 lo = fma2(make_float2(sv[c], sv[c + 1]), sc2, make_float2(b4.x, b4.y));
            const float2 hi = fma2(make_float2(sv[c + 2], sv[c + 3]), sc2, make_float2(b4.z, b4.w));
            sv[c] = lo.x;
            sv[c + 1] = lo.y;
            sv[c + 2] = hi.x;
            sv[c + 3] = hi.y;
            const int m = (c >> 2) & 1;
            mx[m] = max3(mx[m], lo.x, lo.y);
            mx[2 + m] = max3(mx[2 + m], hi.x, hi.y);
          }
        } else {
#pragma unroll
          for (int c = 0; c < NK; ++c) {
            if (c < NK / 2 || !half) {
              sv[c] = c < valid ? fmaf(sv[c], a.sc, bias[c]) : -INFINITY;
              mx[c & 3] = fmaxf(mx[c & 3], sv[c]);
            }
          }
        }
        mbar_arrive(bias_empty + sb);
        const float mt = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
        float alpha = 1.f;
        bool resc = false;
        if (mt > m_run + kRescaleNat) {  // first tile, or the max grew by more than 2^8
          alpha = ex2((m_run - mt) * kLog2e);
          resc = j > 0;
          m_run = mt;
        }
        // every key seen so far masked (groups without a real key): weights 0
        const float neg_m2 = m_run > -INFINITY ? -m_run * kLog2e : 0.f;
        // four partial sums (columns c mod 4), as packed pairs
        const float2 l2e = make_float2(kLog2e, kLog2e), nm2 = make_float2(neg_m2, neg_m2);
        float2 ls01 = make_float2(0.f, 0.f), ls23 = make_float2(0.f, 0.f);
#pragma unroll
        for (int c = 0; c < NK; c += 4) {
          if (c < NK / 2 || !half) {
            const float2 x0 = fma2(make_float2(sv[c], sv[c + 1]), l2e, nm2);
            const float2 x1 = fma2(make_float2(sv[c + 2], sv[c + 3]), l2e, nm2);
            sv[c] = ex2(x0.x);
            sv[c + 1] = ex2(x0.y);
            sv[c + 2] = ex2(x1.x);
            sv[c + 3] = ex2(x1.y);
            ls01 = add2(ls01, make_float2(sv[c], sv[c + 1]));
            ls23 = add2(ls23, make_float2(sv[c + 2], sv[c + 3]));
          }
        }
        l_run = l_run * alpha + ((ls01.x + ls01.y) + (ls23.x + ls23.y));
        if (__any_sync(0xffffffffu, resc)) {
          // O is stable once the previous tile's P Y is done
          ok = mbar_wait(pv_done + ((T - 1) & 1), ((T - 1) >> 1) & 1, abort_flag, a.status);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
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
        // P (bf16 pairs) over the first NK/2 columns of this tile's S buffer
#pragma unroll
        for (int c = 0; c < NK / 32; ++c) {
          if (c == 0 || !half) {
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e)
              pk[e] = pack_bf16x2(sv[c * 32 + 2 * e], sv[c * 32 + 2 * e + 1]);
            tmem_st16(tmem_s(sb) + lane_off + c * 16, pk);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(p_full + sb);
      }
      if (!ok) break;
      // ---- epilogue: O / l -> global rows ----
      ok = mbar_wait(pv_done + ((T - 1) & 1), ((T - 1) >> 1) & 1, abort_flag, a.status);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      ko_epilogue<D>(tmem_o, lane_off, row, 1.f / l_run, sP,
                     out_tile(a, it.g, it.i, it.row0, D), out_stride(a, D),
                     it.nrows, o_empty);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// L-update + output when every row's keys fit one tile (nk = b1*c2 <= NK <=
// 128): the softmax is exact in two passes over the S tile (max, then
// exponentials), so there is no running max and no rescaling of O.  Each
// ring has one slot; S of the next item goes out as soon as the previous
// P Y product has consumed its P (which overwrites S in TMEM), so it
// overlaps the previous item's epilogue.  Warp roles as in ko_kernel; items
// are walked in order, so every barrier's phase is the item counter n.
//   q_full/q_empty, kt_full/kt_empty, y_full/y_empty   operand slots
//   bias_full/bias_empty   entropy bias      s_full   S ready
//   p_full                 P written         pv_done  O = P Y complete
//   o_empty                epilogue has read O
// ---------------------------------------------------------------------------
template <int D, int NK>
struct KO1Layout {
  static constexpr int kQBytes = D / 64 * kRows * 128;
  static constexpr int kTileBytes = D / 64 * NK * 128;  // Kt or Y
  static constexpr int kKtOff = kQBytes;
  static constexpr int kYOff = kKtOff + kTileBytes;
  static constexpr int kPOff = kYOff + kTileBytes;      // epilogue staging, 128 rows x 128 B
  static constexpr int kBiasOff = kPOff + kRows * 128;
  static constexpr int kBarOff = kBiasOff + NK * 4;
  static constexpr int kBytes = kBarOff + 16 * 8;
  static constexpr int kAlloc = kBytes > 100 * 1024 ? kBytes : 100 * 1024;  // <= 2 CTAs / SM
  static constexpr uint32_t kTmemCols = 256;  // O: D columns, S: NK columns
  static_assert(D % 64 == 0 && NK % 64 == 0 && NK <= 128 && D + NK <= 256, "tile sizes");
  static_assert(2 * (kAlloc + 1024) <= 233472, "two CTAs per SM");
};

template <int D, int NK>
__global__ void __launch_bounds__(192, 2)
    ko1_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kt,
               const __grid_constant__ CUtensorMap tm_y, KOArgs a) {
  using L = KO1Layout<D, NK>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (smem_u32(smem) & 1023u) {
    if (tid == 0) atomicExch(a.status, 2);
    return;
  }
  pdl_launch_dependents();
  uint8_t* sQ = smem;
  uint8_t* sKt = smem + L::kKtOff;
  uint8_t* sY = smem + L::kYOff;
  uint8_t* sP = smem + L::kPOff;
  float* sBias = reinterpret_cast<float*>(smem + L::kBiasOff);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* kt_full = bars + 2;
  uint64_t* kt_empty = bars + 3;
  uint64_t* y_full = bars + 4;
  uint64_t* y_empty = bars + 5;
  uint64_t* s_full = bars + 6;
  uint64_t* p_full = bars + 7;
  uint64_t* pv_done = bars + 8;
  uint64_t* bias_full = bars + 9;
  uint64_t* bias_empty = bars + 10;
  uint64_t* o_empty = bars + 11;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 12);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 13);

  if (tid == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    mbar_init(kt_full, 1);
    mbar_init(kt_empty, 1);
    mbar_init(y_full, 1);
    mbar_init(y_empty, 1);
    mbar_init(s_full, 1);
    mbar_init(p_full, 128);
    mbar_init(pv_done, 1);
    mbar_init(bias_full, 32);
    mbar_init(bias_empty, 128);
    mbar_init(o_empty, 128);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tmem_o = tmem;      // columns [0, D)
  const uint32_t tmem_s = tmem + D;  // columns [D, D + NK); P (bf16 pairs) over its first NK/2

  if (warp == 0) {
    // ------------------------- producer: Q, Kt + bias, Y -------------------------
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_kt);
      tma_prefetch_desc(&tm_y);
    }
    bool ok = true;
    long n = 0;
    for (int item = blockIdx.x; item < a.n_items && ok; item += gridDim.x) {
      KOItem it;
      if (!ko_decode<NK>(a, item, it)) continue;
      if (lane == 0) {
        if (n >= 1) ok = mbar_wait(q_empty, (n - 1) & 1, abort_flag, a.status);
        if (ok) {
          const int2 qyz = q_slab_yz(a.tr, it.g, a.b1, a.b2, it.i, it.row0);
          mbar_arrive_expect_tx(q_full, L::kQBytes);
#pragma unroll
          for (int c = 0; c < D / 64; ++c)
            tma_load_3d(sQ + c * kRows * 128, &tm_q, q_full, c * 64, qyz.x, qyz.y);
        }
      }
      if (n == 0) pdl_wait();  // Kt, Y and the bias come from the previous kernel
      if (lane == 0) {
        if (ok && n >= 1) ok = mbar_wait(kt_empty, (n - 1) & 1, abort_flag, a.status);
        if (ok) {
          mbar_arrive_expect_tx(kt_full, L::kTileBytes);
#pragma unroll
          for (int c = 0; c < D / 64; ++c)
            tma_load_2d(sKt + c * NK * 128, &tm_kt, kt_full, c * 64, (int)it.key_row0);
        }
        if (ok && n >= 1) ok = mbar_wait(bias_empty, (n - 1) & 1, abort_flag, a.status);
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      // the entropy bias of the item's nk keys (columns past nk stay stale; masked)
      for (int e = lane; e < a.nk; e += 32) cp_async_4(sBias + e, a.hs + it.key_row0 + e);
      cp_async_arrive_noinc(bias_full);
      if (lane == 0) {
        if (n >= 1) ok = mbar_wait(y_empty, (n - 1) & 1, abort_flag, a.status);
        if (ok) {
          mbar_arrive_expect_tx(y_full, L::kTileBytes);
#pragma unroll
          for (int c = 0; c < D / 64; ++c)
            tma_load_2d(sY + c * NK * 128, &tm_y, y_full, c * 64, (int)it.key_row0);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      ++n;
    }
    if (lane == 0 && *abort_flag && n >= 1) {  // drain this warp's loads (bounded)
      drain(q_full, (n - 1) & 1);
      drain(kt_full, (n - 1) & 1);
      drain(y_full, (n - 1) & 1);
    }
  } else if (warp == 1) {
    // -------------------------------- MMA ---------------------------------
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16(kRows, NK, false);
      const uint32_t idesc_o = idesc_bf16(kRows, D, true);
      const uint64_t dq = desc_kmajor(smem_u32(sQ));
      const uint64_t dkt = desc_kmajor(smem_u32(sKt));
      const uint64_t dy = desc_mnmajor(smem_u32(sY), NK * 128);
      const int kk_pv = (a.nk + 15) / 16;  // P Y over the valid keys only
      bool ok = true;
      long n = 0, issued_s = 0, issued_pv = 0;
      for (int item = blockIdx.x; item < a.n_items && ok; item += gridDim.x) {
        KOItem it;
        if (!ko_decode<NK>(a, item, it)) continue;
        ok = mbar_wait(q_full, n & 1, abort_flag, a.status) &&
             mbar_wait(kt_full, n & 1, abort_flag, a.status) &&
             (n == 0 || mbar_wait(pv_done, (n - 1) & 1, abort_flag, a.status));
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_bf16_ss(tmem_s, dq + (((kk >> 2) * (kRows * 128) + (kk & 3) * 32) >> 4),
                      dkt + (((kk >> 2) * (NK * 128) + (kk & 3) * 32) >> 4), idesc_s,
                      kk > 0 ? 1u : 0u);
        mma_commit(s_full);
        mma_commit(kt_empty);
        mma_commit(q_empty);
        issued_s = n + 1;
        ok = mbar_wait(p_full, n & 1, abort_flag, a.status) &&
             mbar_wait(y_full, n & 1, abort_flag, a.status) &&
             (n == 0 || mbar_wait(o_empty, (n - 1) & 1, abort_flag, a.status));
        if (!ok) break;
        tc_fence_after();
        for (int kk = 0; kk < kk_pv; ++kk)  // A = P from TMEM: 8 columns per 16 keys
          mma_bf16_ts(tmem_o, tmem_s + kk * 8, dy + ((kk * 16 * 128) >> 4), idesc_o,
                      kk > 0 ? 1u : 0u);
        mma_commit(pv_done);
        mma_commit(y_empty);
        issued_pv = n + 1;
        ++n;
      }
      if (*abort_flag) {  // drain this thread's MMAs (bounded)
        if (issued_s > 0) drain(s_full, (issued_s - 1) & 1);
        if (issued_pv > 0) drain(pv_done, (issued_pv - 1) & 1);
      }
    }
    __syncwarp();
  } else {
    // ------------------------- softmax + epilogue --------------------------
    const int quad = warp & 3;
    const int row = quad * 32 + lane;  // TMEM lane == tile row
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const int nch = (a.nk + 31) / 32;  // 32-column chunks holding valid keys
    const float sc = a.sc;
    bool ok = true;
    long n = 0;
    for (int item = blockIdx.x; item < a.n_items && ok; item += gridDim.x) {
      KOItem it;
      if (!ko_decode<NK>(a, item, it)) continue;
      ok = mbar_wait(s_full, n & 1, abort_flag, a.status);
      if (ok) ok = mbar_wait(bias_full, n & 1, abort_flag, a.status);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      // logits sc q.Kt + Hs over the valid keys (one TMEM read, packed pairs
      // with the scalar roundings), then the row max
      float sv[NK];
#pragma unroll
      for (int c = 0; c < NK / 32; ++c) {
        if (c < nch) {
          float t[32];
          tmem_ld32(tmem_s + lane_off + c * 32, t);
#pragma unroll
          for (int e = 0; e < 32; ++e) sv[c * 32 + e] = t[e];
        }
      }
      tmem_wait_ld();
      float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
      const float2 sc2 = make_float2(sc, sc);
#pragma unroll
      for (int c = 0; c < NK; c += 4) {
        if (c < nch * 32) {
          const float4 b4 = *reinterpret_cast<const float4*>(sBias + c);
          float2 lo = fma2(make_float2(sv[c], sv[c + 1]), sc2, make_float2(b4.x, b4.y));
          float2 hi = fma2(make_float2(sv[c + 2], sv[c + 3]), sc2, make_float2(b4.z, b4.w));
          sv[c] = c < a.nk ? lo.x : -INFINITY;
          sv[c + 1] = c + 1 < a.nk ? lo.y : -INFINITY;
          sv[c + 2] = c + 2 < a.nk ? hi.x : -INFINITY;
          sv[c + 3] = c + 3 < a.nk ? hi.y : -INFINITY;
          const int mm = (c >> 2) & 1;
          mx[mm] = max3(mx[mm], sv[c], sv[c + 1]);
          mx[2 + mm] = max3(mx[2 + mm], sv[c + 2], sv[c + 3]);
        }
      }
      const float m = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
      const float neg_m2 = -m * kLog2e;
      // P = exp(S - m) as bf16 pairs over the first columns of S (already
      // read), and the row sum (partial sums over columns c mod 4)
      const float2 l2e = make_float2(kLog2e, kLog2e), nm2 = make_float2(neg_m2, neg_m2);
      float2 ls01 = make_float2(0.f, 0.f), ls23 = ls01;
#pragma unroll
      for (int c = 0; c < NK; c += 4) {
        if (c < nch * 32) {
          const float2 x0 = fma2(make_float2(sv[c], sv[c + 1]), l2e, nm2);
          const float2 x1 = fma2(make_float2(sv[c + 2], sv[c + 3]), l2e, nm2);
          sv[c] = ex2(x0.x);
          sv[c + 1] = ex2(x0.y);
          sv[c + 2] = ex2(x1.x);
          sv[c + 3] = ex2(x1.y);
          ls01 = add2(ls01, make_float2(sv[c], sv[c + 1]));
          ls23 = add2(ls23, make_float2(sv[c + 2], sv[c + 3]));
        }
      }
#pragma unroll
      for (int c = 0; c < NK / 32; ++c) {
        if (c < nch) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) pk[e] = pack_bf16x2(sv[c * 32 + 2 * e], sv[c * 32 + 2 * e + 1]);
          tmem_st16(tmem_s + lane_off + c * 16, pk);
        }
      }
      mbar_arrive(bias_empty);
      const float l_row = (ls01.x + ls01.y) + (ls23.x + ls23.y);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(p_full);
      // ---- epilogue: O / l -> global rows ----
      ok = mbar_wait(pv_done, n & 1, abort_flag, a.status);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      ko_epilogue<D>(tmem_o, lane_off, row, 1.f / l_row, sP,
                     out_tile(a, it.g, it.i, it.row0, D), out_stride(a, D),
                     it.nrows, o_empty);
      ++n;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Step-one aggregated queries under the uniform initial L (bf16):
// Qt0[g][p][i][:] = mean_{l in p} q_(l,i).  One block per (g, p, i): 16-byte
// column chunks x row lanes, every row load of a thread in flight at once;
// the row lanes are summed in a fixed order (warp shuffles, then the NT / 32
// warps through shared memory).  NT = 256 threads while the blocks fit one
// wave (5 per SM), else 128: more, smaller blocks resident at once (measured:
// the 16K-token sweep's 1536 blocks 17.6 -> 13.1 us, the 480p latent's 624
// blocks 0.9 us slower at 128).  Launched with programmatic stream serialisation:
// its blocks may be scheduled while the previous kernel of the stream
// finishes, but they wait for it before reading q (which may be that
// kernel's output) and only then let the next kernel launch, so every later
// kernel of the call (which reads K and V early) runs after all earlier work.
// ---------------------------------------------------------------------------
template <int D, int NT>
__global__ void __launch_bounds__(NT)
    init_qt_bf16_kernel(const bf16* __restrict__ q, bf16* __restrict__ qt0, Problem pb) {
  constexpr int CH = D / 8;        // 16-byte chunks per row
  constexpr int RL = NT / CH;      // row lanes
  __shared__ float red[NT / 32][D];
  const int b1 = pb.b1, b2 = pb.b2, c1 = pb.c1;
  int bid = blockIdx.x;
  const int i = bid % b2;
  bid /= b2;
  const int p = bid % c1;
  const long g = bid / c1;
  int l0 = group_start(b1, c1, p), l1 = group_start(b1, c1, p + 1);
  real_rows(pb, i, l0, l1, &l0, &l1);  // the group's real rows at position i
  pdl_wait();
  pdl_launch_dependents();
  const int ch = threadIdx.x % CH, rl = threadIdx.x / CH, lane = threadIdx.x & 31;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  const uint4* base = reinterpret_cast<const uint4*>(q + token_row(pb, g, 0, i) * D) + ch;
  const long row_stride = (pb.tr ? (long)D : (long)b2 * D) / 8;  // rows l apart, in uint4
#pragma unroll 8
  for (int l = l0 + rl; l < l1; l += RL) {
    const uint4 u = __ldg(base + l * row_stride);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      acc[2 * e] += __uint_as_float(w[e] << 16);
      acc[2 * e + 1] += __uint_as_float(w[e] & 0xffff0000u);
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) {
#pragma unroll
    for (int o = CH; o < 32; o <<= 1) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], o);
  }
  if (lane < CH) {
#pragma unroll
    for (int e = 0; e < 8; ++e) red[threadIdx.x >> 5][ch * 8 + e] = acc[e];
  }
  __syncthreads();
  if (threadIdx.x < D) {
    float sum = 0.f;
#pragma unroll
    for (int w8 = 0; w8 < NT / 32; ++w8) sum += red[w8][threadIdx.x];
    qt0[((g * c1 + p) * b2 + i) * D + threadIdx.x] =
        __float2bfloat16_rn(l1 > l0 ? sum / (float)(l1 - l0) : 0.f);
  }
}

// ---------------------------------------------------------------------------
// Arguments of the streaming R-update (krl_kernel, below): for every
// sub-item (g, p, k, q) and tile of 128 positions,
//   S_q = Qt K_q^T / sqrt(d)            K_q: the keys j of column group q of chunk k
//   R = softmax_j(S_q), Hs = entropy      one TMEM lane (row) per thread
//   [Kt | Y] = R [K_q | V_q]
// with Qt the step-one aggregated queries Qt0 (shared by the chunks of a row
// group) or a later step's per-sub-item rows.
// ---------------------------------------------------------------------------
struct KRArgs {
  bf16* kt;   // [G][b2][c1][b1][c2][d]
  bf16* y;
  float* hs;  // [G][b2][c1][b1][c2]
  int b1, b2, c1, c2, write_y;
  float sc_log2;
  int* status;
  int real_lo, real_hi;  // real tokens (padding): keys outside get zero weight
  int n_itiles;          // 128-position tiles per sub-item (b2 > 128 takes several)
  int tr;                // token order of k and v (see Problem)
  // 0: step one, the aggregated queries Qt0 [G][c1][b2][d] of a row group;
  // 1: later steps, every sub-item (g, p, k, q) has its own rows
  // Qt [G][b1][c1][c2][b2][d]
  int qt_per_item;
};

// First query row (in the tensor map of Qt0 or Qt) of sub-item (g, p, k, q).
__device__ __forceinline__ int kr_qrow(const KRArgs& a, int g, int p, int k, int q) {
  return a.qt_per_item ? (((g * a.b1 + k) * a.c1 + p) * a.c2 + q) * a.b2 : (g * a.c1 + p) * a.b2;
}

// Keys [*j_lo, *j_hi) of the nq keys of column group q (first key js) of
// chunk k are real; an empty range marks a group without a real key.
__device__ __forceinline__ void real_keys(int real_lo, int real_hi, int b2, int k, int js, int nq,
                                          int* j_lo, int* j_hi) {
  const long first = (long)k * b2 + js;
  *j_lo = (int)max(0L, min((long)nq, real_lo - first));
  *j_hi = (int)max((long)*j_lo, min((long)nq, real_hi - first));
}

// Softmax of one R row held as NQ raw logits in sv (this thread's TMEM lane):
// columns [jlo, jhi) are the group's real keys (nq of them without padding).
// On return sv holds exp2(s - m) in log2 units (0 outside the real keys),
// z their sum and t2 = sum exp2(s - m) (s - m), the entropy's numerator.  A
// group without a real key gets all zeros and z = 0.  The unpadded case
// (jlo = 0, jhi = nq: warp-uniform) keeps the single bound check.
template <int NQ>
__device__ __forceinline__ void r_row_softmax(float (&sv)[NQ], float sc_log2, int jlo, int jhi,
                                              int nq, float& z, float& t2) {
  float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
  float zs[4] = {0.f, 0.f, 0.f, 0.f}, ts[4] = {0.f, 0.f, 0.f, 0.f};
  if (jlo == 0 && jhi == nq) {
    // packed pairs (the scalar roundings, half the instructions); the sums
    // over columns j mod 4 are the pairs (0, 1) and (2, 3)
    static_assert(NQ % 4 == 0, "group tile");
    const float2 s2 = make_float2(sc_log2, sc_log2);
#pragma unroll
    for (int j = 0; j < NQ; j += 4) {
      const float2 a = mul2(make_float2(sv[j], sv[j + 1]), s2);
      const float2 b = mul2(make_float2(sv[j + 2], sv[j + 3]), s2);
      sv[j] = j < nq ? a.x : -INFINITY;
      sv[j + 1] = j + 1 < nq ? a.y : -INFINITY;
      sv[j + 2] = j + 2 < nq ? b.x : -INFINITY;
      sv[j + 3] = j + 3 < nq ? b.y : -INFINITY;
      const int m = (j >> 2) & 1;
      mx[m] = max3(mx[m], sv[j], sv[j + 1]);
      mx[2 + m] = max3(mx[2 + m], sv[j + 2], sv[j + 3]);
    }
    const float m2 = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
    const float2 nm = make_float2(-m2, -m2);
    float2 z01 = make_float2(0.f, 0.f), z23 = z01, t01 = z01, t23 = z01;
#pragma unroll
    for (int j = 0; j < NQ; j += 4) {
      const float2 d0 = add2(make_float2(sv[j], sv[j + 1]), nm);  // -inf for j >= nq
      const float2 d1 = add2(make_float2(sv[j + 2], sv[j + 3]), nm);
      sv[j] = ex2(d0.x);
      sv[j + 1] = ex2(d0.y);
      sv[j + 2] = ex2(d1.x);
      sv[j + 3] = ex2(d1.y);
      const float2 e0 = make_float2(sv[j], sv[j + 1]), e1 = make_float2(sv[j + 2], sv[j + 3]);
      z01 = add2(z01, e0);
      z23 = add2(z23, e1);
      const float2 p0 = mul2(e0, d0), p1 = mul2(e1, d1);
      t01 = add2(t01, make_float2(j < nq ? p0.x : 0.f, j + 1 < nq ? p0.y : 0.f));
      t23 = add2(t23, make_float2(j + 2 < nq ? p1.x : 0.f, j + 3 < nq ? p1.y : 0.f));
    }
    z = (z01.x + z01.y) + (z23.x + z23.y);
    t2 = (t01.x + t01.y) + (t23.x + t23.y);
    return;
  } else {
#pragma unroll
    for (int j = 0; j < NQ; ++j) {
      sv[j] = (j >= jlo && j < jhi) ? sv[j] * sc_log2 : -INFINITY;
      mx[j & 3] = fmaxf(mx[j & 3], sv[j]);
    }
    // a group without a real key has no finite logit: its weights become 0
    const float m2 = jhi > jlo ? fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) : 0.f;
#pragma unroll
    for (int j = 0; j < NQ; ++j) {
      const float d2 = sv[j] - m2;  // -inf outside the real keys
      sv[j] = ex2(d2);
      zs[j & 3] += sv[j];
      ts[j & 3] += (j >= jlo && j < jhi) ? sv[j] * d2 : 0.f;
    }
  }
  z = (zs[0] + zs[1]) + (zs[2] + zs[3]);
  t2 = (ts[0] + ts[1]) + (ts[2] + ts[3]);
}

// ---------------------------------------------------------------------------
// R-update for column groups of more than 128 keys, persistent and
// warp-specialised.  A work item is (g, k, p, position tile, group q): 128
// aggregated queries against the group's keys, streamed in 128-key tiles
// with an online softmax (thread = row, log2 units):
//   S_j = Qt K_j^T                     128 x 128 in TMEM, two buffers
//   m, z, T = sum e (s - m)            running per row; when a tile's max
//                                      exceeds m by more than 2^8 (lazy), m
//                                      moves and z, T and the accumulator
//                                      rows are scaled by 2^(m_old - m_new)
//   P_j = 2^(s sc log2(e) - m)         bf16 pairs written over S_j in TMEM
//   [Kt | Y] += P_j [K_j | V_j]          128 x 2d in TMEM, A = P_j from TMEM
// then [Kt | Y] / z and Hs = ln z - ln 2 T / z.  Warp 0 loads the query
// tile and the K_j | V_j tiles (TMA, a two-slot ring), warp 1 issues the
// MMAs from one thread (event-driven, as the output kernel), and warps 2-9
// run the softmax and the epilogue, two warps per row: warps 2-5 take keys
// 0-63 of every tile, warps 6-9 keys 64-127.  The two halves exchange each
// tile's row maxima through shared memory, so both hold the same running
// maximum and take the same rescaling decisions; each keeps its own z and T
// (added once per item) and rescales its half of the accumulator columns.
// In the epilogue each warp stores its 32 rows of every other 64-column
// block through a 4-D box clipped at b2.  S_{j+1} is computed while the
// softmax works on S_j, and the next item's first tiles while the epilogue
// stores this one's rows.  Barriers (tile counter T over the CTA's items):
//   q_full / q_empty         query tile of an item
//   kv_full / kv_empty [2]   K_j | V_j ring (free once P_j [K_j | V_j] is done)
//   s_full [2]               S_j in its TMEM buffer
//   p_full [2]               P_j written over S_j
//   pv_done [2]              the product of tile j complete (its buffer free)
//   o_empty                  the epilogue has read the accumulator
//   xchg [2]                 both halves' tile maxima are in shared memory
//   zx                       both halves' z (and T) of an item are in shared memory
// ---------------------------------------------------------------------------
template <int D>
struct KRLLayout {
  static constexpr int kChunk = kRows * 128;                  // 128 rows x 64 bf16
  static constexpr int kQOff = 0;                             // D / 64 chunks
  static constexpr int kSlotBytes = 2 * (D / 64) * kChunk;    // K chunks, then V chunks
  static constexpr int kKVOff = D / 64 * kChunk;              // two slots
  static constexpr int kStageOff = kKVOff + 2 * kSlotBytes;   // two chunks: 64 columns each
  static constexpr int kXchgOff = kStageOff + 2 * kChunk;     // float [2][2][kRows] maxima
  static constexpr int kZOff = kXchgOff + 4 * kRows * 4;      // float [2][3][kRows]: z, z, T
  static constexpr int kBarOff = kZOff + 6 * kRows * 4;
  static constexpr int kBytes = kBarOff + 20 * 8;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kSCol = 2 * D;  // S buffers at [2d, 2d + 128), [2d + 128, 2d + 256)
  static_assert(2 * D + 256 <= 512 && kBytes <= 227 * 1024, "TMEM and shared memory");
};

struct KRLItem {
  int g, k, p, q, i0, js, nq, n_sub, jlo, jhi;
};

// Item order: group q fastest, then position tile, row group, chunk, head.
__device__ __forceinline__ void krl_decode(const KRArgs& a, int item, KRLItem& t) {
  int bid = item;
  t.q = bid % a.c2;
  bid /= a.c2;
  const int it = bid % a.n_itiles;
  bid /= a.n_itiles;
  t.p = bid % a.c1;
  bid /= a.c1;
  t.k = bid % a.b1;
  t.g = bid / a.b1;
  t.i0 = it * kRows;
  t.js = group_start(a.b2, a.c2, t.q);
  t.nq = group_start(a.b2, a.c2, t.q + 1) - t.js;
  t.n_sub = (t.nq + 127) / 128;
  real_keys(a.real_lo, a.real_hi, a.b2, t.k, t.js, t.nq, &t.jlo, &t.jhi);
}

__device__ __forceinline__ int krl_nsub(const KRArgs& a, int item) {
  const int q = item % a.c2;
  return (group_start(a.b2, a.c2, q + 1) - group_start(a.b2, a.c2, q) + 127) / 128;
}

template <int D>
__global__ void __launch_bounds__(320, 1)
    krl_kernel(const __grid_constant__ CUtensorMap tm_qt, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_kt,
               const __grid_constant__ CUtensorMap tm_y, KRArgs a, int n_items) {
  using L = KRLLayout<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (smem_u32(smem) & 1023u) {
    if (tid == 0) atomicExch(a.status, 2);
    return;
  }
  pdl_launch_dependents();
  uint8_t* sQ = smem + L::kQOff;
  auto sKV = [&](int sl) { return smem + L::kKVOff + sl * L::kSlotBytes; };
  uint8_t* sStage = smem + L::kStageOff;
  float* sXchg = reinterpret_cast<float*>(smem + L::kXchgOff);
  float* sZ = reinterpret_cast<float*>(smem + L::kZOff);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* kv_full = bars + 2;   // [2]
  uint64_t* kv_empty = bars + 4;  // [2]
  uint64_t* s_full = bars + 6;    // [2]
  uint64_t* p_full = bars + 8;    // [2]
  uint64_t* pv_done = bars + 10;  // [2]
  uint64_t* o_empty = bars + 12;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 13);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 14);
  uint64_t* xchg = bars + 15;     // [2]
  uint64_t* zx = bars + 17;
  if (tid == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(kv_full + s, 1);
      mbar_init(kv_empty + s, 1);
      mbar_init(s_full + s, 1);
      mbar_init(p_full + s, 256);
      mbar_init(pv_done + s, 1);
      mbar_init(xchg + s, 256);
    }
    mbar_init(o_empty, 256);
    mbar_init(zx, 256);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;  // accumulator [Kt | Y] in columns [0, 2d)
  auto tmem_s = [&](int sb) { return tmem + L::kSCol + sb * 128; };

  if (warp == 0) {
    // ---------------------------- producer ----------------------------
    if (lane == 0) {
      tma_prefetch_desc(&tm_qt);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      pdl_wait();  // the queries come from the previous kernel
      long T = 0, last_kv = -1;
      int q_loads = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
        KRLItem t;
        krl_decode(a, item, t);
        if (q_loads >= 1) ok = mbar_wait(q_empty, (q_loads - 1) & 1, abort_flag, a.status);
        if (!ok) break;
        mbar_arrive_expect_tx(q_full, (D / 64) * L::kChunk);
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          tma_load_2d(sQ + c * L::kChunk, &tm_qt, q_full, c * 64,
                      kr_qrow(a, t.g, t.p, t.k, t.q) + t.i0);
        ++q_loads;
        for (int j = 0; j < t.n_sub && ok; ++j, ++T) {
          const int sl = (int)(T & 1);
          if (T >= 2) ok = mbar_wait(kv_empty + sl, ((T >> 1) - 1) & 1, abort_flag, a.status);
          if (!ok) break;
          mbar_arrive_expect_tx(kv_full + sl, L::kSlotBytes);
          const int2 kyz = kv_yz(a.tr, t.g, a.b1, a.b2, t.k, t.js + j * 128);
#pragma unroll
          for (int c = 0; c < D / 64; ++c) {
            tma_load_3d(sKV(sl) + c * L::kChunk, &tm_k, kv_full + sl, c * 64, kyz.x, kyz.y);
            tma_load_3d(sKV(sl) + (D / 64 + c) * L::kChunk, &tm_v, kv_full + sl, c * 64, kyz.x,
                        kyz.y);
          }
          last_kv = T;
        }
      }
      if (*abort_flag) {  // drain the loads this thread issued (bounded)
        if (q_loads >= 1) drain(q_full, (q_loads - 1) & 1);
        for (long t = (last_kv >= 1 ? last_kv - 1 : 0); t <= last_kv; ++t)
          drain(kv_full + (t & 1), (t >> 1) & 1);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------- MMA --------------------------------
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16(kRows, 128, false);
      const uint32_t idesc_o = idesc_bf16(kRows, 2 * D, true);
      const uint64_t dq = desc_kmajor(smem_u32(sQ));
      const uint64_t dk0 = desc_kmajor(smem_u32(sKV(0))), dk1 = desc_kmajor(smem_u32(sKV(1)));
      const uint64_t dkv0 = desc_mnmajor(smem_u32(sKV(0)), L::kChunk),
                     dkv1 = desc_mnmajor(smem_u32(sKV(1)), L::kChunk);
      int s_item = blockIdx.x, p_item = blockIdx.x;
      int s_nsub = s_item < n_items ? krl_nsub(a, s_item) : 0;
      int p_nsub = s_nsub;
      int s_j = 0, s_n = 0, p_j = 0, p_n = 0;
      long Ts = 0, Tp = 0, last_s = -1, last_pv = -1;
      bool ok = true;
      unsigned long long idle_since = global_ns();
      while (p_item < n_items && ok) {
        bool progressed = false;
        if (s_item < n_items) {
          const int st = (int)(Ts & 1);
          if ((s_j > 0 || mbar_test(q_full, s_n & 1)) && mbar_test(kv_full + st, (Ts >> 1) & 1) &&
              (Ts < 2 || mbar_test(pv_done + st, ((Ts >> 1) - 1) & 1))) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
              mma_bf16_ss(tmem_s(st), dq + (((kk >> 2) * L::kChunk + (kk & 3) * 32) >> 4),
                          (st ? dk1 : dk0) + (((kk >> 2) * L::kChunk + (kk & 3) * 32) >> 4),
                          idesc_s, kk > 0 ? 1u : 0u);
            mma_commit(s_full + st);
            last_s = Ts;
            ++Ts;
            if (++s_j == s_nsub) {
              mma_commit(q_empty);  // the item's query tile is no longer needed
              s_j = 0;
              ++s_n;
              s_item += gridDim.x;
              s_nsub = s_item < n_items ? krl_nsub(a, s_item) : 0;
            }
            progressed = true;
          }
        }
        if (Tp < Ts) {
          const int st = (int)(Tp & 1);
          if (mbar_test(p_full + st, (Tp >> 1) & 1) &&
              (p_j > 0 || p_n == 0 || mbar_test(o_empty, (p_n - 1) & 1))) {
            tc_fence_after();
            // A = P_j from TMEM (8 columns per 16 keys), B = [K_j | V_j] MN-major
#pragma unroll
            for (int kk = 0; kk < 128 / 16; ++kk)
              mma_bf16_ts(tmem, tmem_s(st) + kk * 8, (st ? dkv1 : dkv0) + ((kk * 16 * 128) >> 4),
                          idesc_o, (p_j > 0 || kk > 0) ? 1u : 0u);
            mma_commit(kv_empty + st);
            mma_commit(pv_done + st);
            last_pv = Tp;
            ++Tp;
            if (++p_j == p_nsub) {
              p_j = 0;
              ++p_n;
              p_item += gridDim.x;
              p_nsub = p_item < n_items ? krl_nsub(a, p_item) : 0;
            }
            progressed = true;
          }
        }
        if (progressed) {
          idle_since = global_ns();
        } else if ((__nanosleep(20), *abort_flag)) {
          ok = false;
        } else if (global_ns() - idle_since > kWaitLimitNs) {
          *abort_flag = 1;
          atomicExch(a.status, 1);
          ok = false;
        }
      }
      if (*abort_flag) {  // drain this thread's MMAs (bounded)
        if (last_s >= 0) drain(s_full + (last_s & 1), (last_s >> 1) & 1);
        if (last_pv >= 0) drain(pv_done + (last_pv & 1), (last_pv >> 1) & 1);
      }
    }
    __syncwarp();
  } else {
    // -------------- softmax (two warps per row) + epilogue --------------
    const int half = (warp - 2) >> 2;  // 0: keys 0-63 of a tile (warps 2-5), 1: keys 64-127
    const int quad = warp & 3;
    const int r = quad * 32 + lane;  // TMEM lane == tile row == position i0 + r
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    long T = 0;
    int n_done = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
      KRLItem t;
      krl_decode(a, item, t);
      float m = -INFINITY, z = 0.f, t2 = 0.f;  // m shared by both halves; z, t2 this half's
      for (int j = 0; j < t.n_sub; ++j, ++T) {
        const int sb = (int)(T & 1);
        ok = mbar_wait(s_full + sb, (T >> 1) & 1, abort_flag, a.status);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        const int k0 = j * 128 + half * 64;  // this half's first key of the group
        float sv[64];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          float tt[32];
          tmem_ld32(tmem_s(sb) + lane_off + half * 64 + c * 32, tt);
#pragma unroll
          for (int e = 0; e < 32; ++e) sv[c * 32 + e] = tt[e];
        }
        tmem_wait_ld();
        // logits in log2 units over the group's real keys; 4 partial maxima
        float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        const bool full = t.jlo <= k0 && k0 + 64 <= t.jhi;  // warp-uniform
        if (full) {
          const float2 s2 = make_float2(a.sc_log2, a.sc_log2);
#pragma unroll
          for (int c = 0; c < 64; c += 4) {
            const float2 lo = mul2(make_float2(sv[c], sv[c + 1]), s2);
            const float2 hi = mul2(make_float2(sv[c + 2], sv[c + 3]), s2);
            sv[c] = lo.x;
            sv[c + 1] = lo.y;
            sv[c + 2] = hi.x;
            sv[c + 3] = hi.y;
            const int mm = (c >> 2) & 1;
            mx[mm] = max3(mx[mm], lo.x, lo.y);
            mx[2 + mm] = max3(mx[2 + mm], hi.x, hi.y);
          }
        } else {
#pragma unroll
          for (int c = 0; c < 64; ++c) {
            const int jj = k0 + c;
            sv[c] = (jj >= t.jlo && jj < t.jhi) ? sv[c] * a.sc_log2 : -INFINITY;
            mx[c & 3] = fmaxf(mx[c & 3], sv[c]);
          }
        }
        // the tile maximum of the row: this half's, then the other half's
        // (buffer sb is written again two tiles on, after the other half
        // has passed the next exchange)
        const float mh = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
        float* xb = sXchg + sb * 2 * kRows;
        xb[half * kRows + r] = mh;
        tc_fence_before();  // this half's S loads are done before the other half writes P
        mbar_arrive(xchg + sb);
        ok = mbar_wait(xchg + sb, (T >> 1) & 1, abort_flag, a.status);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        const float mt = fmaxf(mh, xb[(1 - half) * kRows + r]);
        float alpha = 1.f;
        bool resc = false;
        if (mt > m + 8.f) {  // first real keys, or the max grew by more than 2^8
          alpha = m > -INFINITY ? ex2(m - mt) : 0.f;
          t2 = m > -INFINITY ? alpha * (t2 + z * (m - mt)) : 0.f;
          z *= alpha;
          resc = j > 0;
          m = mt;
        }
        if (__any_sync(0xffffffffu, resc)) {
          // the accumulator is stable once the previous tile's product is
          // done; each half scales its d columns of [Kt | Y]
          ok = mbar_wait(pv_done + ((T - 1) & 1), ((T - 1) >> 1) & 1, abort_flag, a.status);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          tc_fence_after();
#pragma unroll 1
          for (int c = half * (D / 32); c < (half + 1) * (D / 32); ++c) {
            float tt[32];
            tmem_ld32(tmem + lane_off + c * 32, tt);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) tt[e] *= alpha;
            tmem_st32(tmem + lane_off + c * 32, tt);
          }
          tmem_wait_st();
        }
        const float base = m > -INFINITY ? m : 0.f;
        float zs[4] = {0.f, 0.f, 0.f, 0.f}, ts[4] = {0.f, 0.f, 0.f, 0.f};
        // exponentials 32 keys at a time, each group's P (bf16 pairs) stored
        // at once: this half's 32 columns of the first 64 of the S buffer
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const float d2 = sv[c * 32 + e] - base;  // -inf outside the real keys
            const float w = ex2(d2);
            zs[e & 3] += w;
            ts[e & 3] += full ? w * d2 : (w > 0.f ? w * d2 : 0.f);
            if (e & 1)
              pk[e >> 1] = pack_bf16x2(sv[c * 32 + e - 1], w);
            else
              sv[c * 32 + e] = w;
          }
          tmem_st16(tmem_s(sb) + lane_off + half * 32 + c * 16, pk);
        }
        z += (zs[0] + zs[1]) + (zs[2] + zs[3]);
        t2 += (ts[0] + ts[1]) + (ts[2] + ts[3]);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(p_full + sb);
      }
      if (!ok) break;
      // ---- epilogue: [Kt | Y] / z; this warp stores its 32 rows of the
      // 64-column blocks cb = half, half + 2, ... ----
      // both halves' z and the second half's T through shared memory (a
      // buffer per item parity, written again after the next exchange)
      float* zb = sZ + (n_done & 1) * 3 * kRows;
      zb[half * kRows + r] = z;
      if (half == 1) zb[2 * kRows + r] = t2;
      mbar_arrive(zx);
      ok = mbar_wait(zx, n_done & 1, abort_flag, a.status);
      if (ok) ok = mbar_wait(pv_done + ((T - 1) & 1), ((T - 1) >> 1) & 1, abort_flag, a.status);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const float zt = zb[r] + zb[kRows + r];  // the same sum in both halves
      const float inv = zt > 0.f ? 1.f / zt : 0.f;
      const int nblk = (a.write_y ? 2 : 1) * (D / 64);
      const int ycoord = (t.p * a.b1 + t.k) * a.c2 + t.q;
      const int iw = t.i0 + quad * 32;  // this warp's first position
      const bool store = iw < a.b2;     // warp-uniform
      uint8_t* buf = sStage + half * L::kChunk + quad * 32 * 128;
#pragma unroll 1
      for (int cb = half; cb < nblk; cb += 2) {
        if (store) {  // the previous store from buf has read it
          if (lane == 0) bulk_wait_read<0>();
          __syncwarp();
        }
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          float tt[32];
          tmem_ld32(tmem + lane_off + cb * 64 + hf * 32, tt);
          tmem_wait_ld();
          if (store) {
#pragma unroll
            for (int uu = 0; uu < 4; ++uu) {
              uint4 pk;
              pk.x = pack_bf16x2(tt[8 * uu + 0] * inv, tt[8 * uu + 1] * inv);
              pk.y = pack_bf16x2(tt[8 * uu + 2] * inv, tt[8 * uu + 3] * inv);
              pk.z = pack_bf16x2(tt[8 * uu + 4] * inv, tt[8 * uu + 5] * inv);
              pk.w = pack_bf16x2(tt[8 * uu + 6] * inv, tt[8 * uu + 7] * inv);
              const int chunk = hf * 4 + uu;
              *reinterpret_cast<uint4*>(buf + lane * 128 + ((chunk ^ (lane & 7)) << 4)) = pk;
            }
          }
        }
        if (store) {
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_4d(cb < D / 64 ? &tm_kt : &tm_y, buf, (cb % (D / 64)) * 64, ycoord, iw, t.g);
            bulk_commit();
          }
        }
      }
      // the accumulator is read out: the next item's first product may overwrite it
      tc_fence_before();
      mbar_arrive(o_empty);
      if (half == 0 && t.i0 + r < a.b2) {
        const float tt2 = t2 + zb[2 * kRows + r];
        const long orow = ((((long)t.g * a.b2 + t.i0 + r) * a.c1 + t.p) * a.b1 + t.k) * a.c2 + t.q;
        a.hs[orow] = zt > 0.f ? logf(zt) - tt2 * 0.69314718055994531f / zt : -INFINITY;
      }
      ++n_done;
    }
    if (lane == 0) bulk_wait<0>();  // stores done reading shared memory before exit
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Persistent R-update for column-group tiles NQ <= 96 (paired tiles: NQ <=
// 64) (step one, and the later steps with per-sub-item queries).  One CTA
// per SM walks a contiguous range of sub-items (g, p, k, q): one item (g, p, k)
// is split into c2 sub-items, one per column group q.  Warp 0 loads (Qt0, and
// K_q / V_q through a ring of slots), warp 1 issues the MMAs, and two
// warpgroups (warps 2-5 and 6-9) take alternate tiles: softmax (R is
// normalised before the MMA), then the Kt / Y rows through TMA bulk stores.
// Each warpgroup owns one 2d-column TMEM slot in which S is later
// overwritten by [Kt | Y], so tile t+1's S and softmax overlap tile t's
// stores.  In the epilogue every warp stores its own 32 rows through a 4-D
// box clipped at b2, staging them in its own rows of P (dead once the
// [Kt | Y] product has read it), with no barrier across the warpgroup.
//
// Paired tiles (PAIR, b2 <= 64): the b2 positions of one sub-item fill only
// half of the 128 TMEM lanes, so a tile carries two consecutive sub-items A
// and B.  Rows 0-63 of the A operand hold sub-item A's aggregated queries and
// rows 64-127 sub-item B's; the key operand stacks A's NQ keys over B's, so S
// is 128 x 2NQ and rows 0-63 use its first NQ columns, rows 64-127 its last
// NQ.  P is block diagonal ([R_A 0; 0 R_B]), so one product with the stacked
// [K | V] of both sub-items gives [Kt | Y] of A in rows 0-63 and of B in rows
// 64-127.
//
// Barriers (tile counter t over the CTA's tiles):
//   q_full / q_empty       Qt0 tile        kv_full / kv_empty   K/V ring
//   s_full[w] / o_full[w]  S / [Kt | Y] of warpgroup w's slot complete
//   p_full[w]              P written       tmem_free[w]         slot read out
// ---------------------------------------------------------------------------
template <int D, int NQ, bool PAIR>
struct KR2Layout {
  static constexpr int kHalves = PAIR ? 2 : 1;             // sub-items per tile
  static constexpr int kKeys = kHalves * NQ;               // N of S, K-extent of [K | V]
  static constexpr int kBox = NQ * 128;                    // one TMA box: NQ keys x 64 columns
  static constexpr int kBlk = kKeys * 128;                 // one 64-column block of K or V
  static constexpr int kKVBytes = 2 * (D / 64) * kBlk;     // K blocks, then V blocks
  // three ring slots when they fit beside Q and P, else two
  static constexpr int kKVSlots =
      PAIR ? 2 : (D / 64 * kRows * 128 + 3 * kKVBytes + 4 * kRows * 128 + 256 <= 227 * 1024 ? 3 : 2);
  // P (K-major, 64-key chunks of 128 rows): two chunks, so that once the
  // [Kt | Y] product has read P each warp finds two 4 KB staging buffers in
  // its own 32 rows for the epilogue's stores.
  static constexpr int kPBytes = 2 * kRows * 128;
  static constexpr int kQOff = 0;
  static constexpr int kKVOff = D / 64 * kRows * 128;
  static constexpr int kPOff = kKVOff + kKVSlots * kKVBytes;       // [2 wg]
  static constexpr int kBarOff = kPOff + 2 * kPBytes;
  static constexpr int kBytes = kBarOff + 32 * 8;
  static_assert(NQ % 16 == 0 && NQ <= (PAIR ? 64 : 96), "group tile");
  static_assert(kBytes <= 227 * 1024, "shared memory");
};

struct KR2Args {
  bf16* kt;   // [G][b2][c1][b1][c2][d]
  bf16* y;
  float* hs;
  int b1, b2, c1, c2, n_items, write_y;
  float sc_log2;
  int* status;
  int real_lo, real_hi;  // real tokens (padding): keys outside get zero weight
  // 0: step one, the aggregated queries Qt0 [G][c1][b2][d] are shared by the
  // chunks k and groups q of a row group; 1: later steps, every sub-item
  // (g, p, k, q) has its own rows Qt [G][b1][c1][c2][b2][d]
  int qt_per_item;
  int tr;  // token order of k and v (see Problem)
};


struct KR2Sub {
  int g, p, k, q, gp;
};

__device__ __forceinline__ KR2Sub kr2_sub(const KR2Args& a, long n_sub) {
  KR2Sub s;
  const int item = (int)(n_sub / a.c2);
  s.q = (int)(n_sub % a.c2);
  s.k = item % a.b1;
  s.gp = item / a.b1;  // g * c1 + p
  s.p = s.gp % a.c1;
  s.g = s.gp / a.c1;
  return s;
}

// First aggregated-query row of a sub-item.
__device__ __forceinline__ long kr2_qrow(const KR2Args& a, const KR2Sub& s) {
  return a.qt_per_item ? ((((long)s.g * a.b1 + s.k) * a.c1 + s.p) * a.c2 + s.q) * a.b2
                       : (long)s.gp * a.b2;
}

// Next sub-item in (gp, k, q) order.
__device__ __forceinline__ void kr2_next(const KR2Args& a, KR2Sub& s) {
  if (++s.q == a.c2) {
    s.q = 0;
    if (++s.k == a.b1) {
      s.k = 0;
      ++s.gp;
      s.p = s.gp % a.c1;
      s.g = s.gp / a.c1;
    }
  }
}

// Which aggregated-query rows a tile needs: (gp of its first sub-item, gp of
// its last); a change of key means a new Qt0 load.
__device__ __forceinline__ long kr2_qkey(int gp_a, int gp_b) {
  return ((long)gp_a << 32) | (unsigned)gp_b;
}

template <int D, int NQ, bool PAIR>
__global__ void __launch_bounds__(320, 1)
    kr2_kernel(const __grid_constant__ CUtensorMap tm_qt, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_kt,
               const __grid_constant__ CUtensorMap tm_y, KR2Args a) {
  using L = KR2Layout<D, NQ, PAIR>;
  constexpr int H = L::kHalves;
  constexpr int kSlots = L::kKVSlots;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (smem_u32(smem) & 1023u) {
    if (tid == 0) atomicExch(a.status, 2);
    return;
  }
  pdl_launch_dependents();
  // this CTA's tiles: H consecutive sub-items each, sub-items [s0, s1)
  const long n_sub = (long)a.n_items * a.c2;
  const long n_units = (n_sub + H - 1) / H;
  const long s0 = n_units * blockIdx.x / gridDim.x * H;
  const long s1 = min(n_units * (blockIdx.x + 1) / gridDim.x * H, n_sub);
  const long ntiles = (s1 - s0 + H - 1) / H;

  uint8_t* sQ = smem + L::kQOff;
  auto sKV = [&](int sl) { return smem + L::kKVOff + sl * L::kKVBytes; };
  auto sP = [&](int w) { return smem + L::kPOff + w * L::kPBytes; };
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* kv_full = bars + 2;    // [kSlots]
  uint64_t* kv_empty = bars + 5;   // [kSlots]
  uint64_t* s_full = bars + 8;     // [2]
  uint64_t* o_full = bars + 10;    // [2]
  uint64_t* p_full = bars + 12;    // [2]
  uint64_t* tmem_free = bars + 14; // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 16);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 17);

  if (tid == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < kSlots; ++i) {
      mbar_init(kv_full + i, 1);
      mbar_init(kv_empty + i, 1);
    }
    for (int w = 0; w < 2; ++w) {
      mbar_init(s_full + w, 1);
      mbar_init(o_full + w, 1);
      mbar_init(p_full + w, 128);
      mbar_init(tmem_free + w, 128);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------ producer ------------------------------
    if (lane == 0) {
      tma_prefetch_desc(&tm_qt);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      long cur_key = -1;
      int nq_loads = 0;
      bool ok = true;
      long last_kv = -1;
      KR2Sub cur = kr2_sub(a, s0);
      for (long t = 0; t < ntiles && ok; ++t) {
        const int sl = (int)(t % kSlots);
        const int nh = (int)min((long)H, s1 - (s0 + t * H));
        if (t >= kSlots) ok = mbar_wait(kv_empty + sl, ((t / kSlots) - 1) & 1, abort_flag, a.status);
        if (!ok) break;
        mbar_arrive_expect_tx(kv_full + sl, H * 2 * (D / 64) * L::kBox);
        const int gp_a = cur.gp;
        int gp_b = gp_a;
        int2 kyz = make_int2(0, 0);
        long qrow[2] = {0, 0};
        for (int h = 0; h < H; ++h) {
          // An absent second half (odd count, last tile) repeats the first:
          // finite keys that its zero rows of P weigh by zero.
          if (h < nh) {
            kyz = kv_yz(a.tr, cur.g, a.b1, a.b2, cur.k, group_start(a.b2, a.c2, cur.q));
            gp_b = cur.gp;
            qrow[h] = kr2_qrow(a, cur);
            kr2_next(a, cur);
          } else {
            qrow[h] = qrow[0];
          }
#pragma unroll
          for (int c = 0; c < D / 64; ++c) {
            tma_load_3d(sKV(sl) + c * L::kBlk + h * L::kBox, &tm_k, kv_full + sl, c * 64, kyz.x,
                        kyz.y);
            tma_load_3d(sKV(sl) + (D / 64 + c) * L::kBlk + h * L::kBox, &tm_v, kv_full + sl,
                        c * 64, kyz.x, kyz.y);
          }
        }
        last_kv = t;
        // a new tile needs new query rows when its row groups change (step
        // one) or always (later steps, one set of rows per sub-item)
        const long key = a.qt_per_item ? t : kr2_qkey(gp_a, gp_b);
        if (key != cur_key) {
          if (nq_loads == 0) pdl_wait();  // the queries come from the previous kernel
          if (ok && nq_loads >= 1) ok = mbar_wait(q_empty, (nq_loads - 1) & 1, abort_flag, a.status);
          if (!ok) break;
          mbar_arrive_expect_tx(q_full, D / 64 * kRows * 128);
          if (PAIR) {
#pragma unroll
            for (int c = 0; c < D / 64; ++c) {
              tma_load_2d(sQ + c * kRows * 128, &tm_qt, q_full, c * 64, (int)qrow[0]);
              tma_load_2d(sQ + c * kRows * 128 + 64 * 128, &tm_qt, q_full, c * 64, (int)qrow[1]);
            }
          } else {
#pragma unroll
            for (int c = 0; c < D / 64; ++c)
              tma_load_2d(sQ + c * kRows * 128, &tm_qt, q_full, c * 64, (int)qrow[0]);
          }
          cur_key = key;
          ++nq_loads;
        }
      }
      if (*abort_flag) {
        if (nq_loads >= 1) drain(q_full, (nq_loads - 1) & 1);
        for (long t = (last_kv >= kSlots - 1 ? last_kv - (kSlots - 1) : 0); t <= last_kv; ++t)
          drain(kv_full + t % kSlots, (t / kSlots) & 1);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // -------------------------------- MMA ---------------------------------
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16(kRows, L::kKeys, false);
      const uint32_t idesc_o = idesc_bf16(kRows, 2 * D, true);
      // Base descriptors, built once; each MMA adds a compile-time offset
      // (in 16-byte units) to the start-address field.  The issuing thread
      // shares its scheduler with softmax warps, so its path is kept short.
      const uint64_t dq = desc_kmajor(smem_u32(sQ));
      const uint64_t dk0 = desc_kmajor(smem_u32(sKV(0))), dk1 = desc_kmajor(smem_u32(sKV(1))),
                     dk2 = desc_kmajor(smem_u32(sKV(kSlots > 2 ? 2 : 1)));
      const uint64_t dkv0 = desc_mnmajor(smem_u32(sKV(0)), L::kBlk),
                     dkv1 = desc_mnmajor(smem_u32(sKV(1)), L::kBlk),
                     dkv2 = desc_mnmajor(smem_u32(sKV(kSlots > 2 ? 2 : 1)), L::kBlk);
      const uint64_t dp0 = desc_kmajor(smem_u32(sP(0))), dp1 = desc_kmajor(smem_u32(sP(1)));
      auto pick3 = [](int i, uint64_t x0, uint64_t x1, uint64_t x2) {
        return i == 0 ? x0 : (i == 1 ? x1 : x2);
      };
      int nq_loads = 0;
      bool ok = true;
      long last_s = -1, last_o = -1;
      // Event-driven issue: S of the next tile and [Kt | Y] of the oldest
      // pending one go out as soon as their inputs are ready, in whichever
      // order that happens, so one warpgroup's epilogue never holds back the
      // other warpgroup's product.  The sub-items are walked incrementally.
      long ts = 0, tp = 0;
      KR2Sub cur = kr2_sub(a, s0);
      long cur_key = -1;
      // key of tile ts (and the walker moved to tile ts + 1)
      auto tile_key = [&](long t) {
        const int nh = (int)min((long)H, s1 - (s0 + t * H));
        const int gp_a = cur.gp;
        int gp_b = gp_a;
        for (int h = 0; h < nh; ++h) {
          gp_b = cur.gp;
          kr2_next(a, cur);
        }
        return a.qt_per_item ? t : kr2_qkey(gp_a, gp_b);
      };
      long key = ntiles > 0 ? tile_key(0) : -1;
      unsigned long long idle_since = global_ns();
      while (tp < ntiles && ok) {
        bool progressed = false;
        if (ts < ntiles) {
          const int w = (int)(ts & 1), sl = (int)(ts % kSlots);
          bool ready = true;
          if (key != cur_key) {
            ready = mbar_test(q_full, nq_loads & 1);
            if (ready) {
              cur_key = key;
              ++nq_loads;
            }
          }
          if (ready && mbar_test(kv_full + sl, (ts / kSlots) & 1) &&
              (ts < 2 || mbar_test(tmem_free + w, ((ts >> 1) - 1) & 1))) {
            tc_fence_after();
            const uint64_t dks = pick3(sl, dk0, dk1, dk2);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
              mma_bf16_ss(tmem + w * 256, dq + (((kk >> 2) * (kRows * 128) + (kk & 3) * 32) >> 4),
                          dks + (((kk >> 2) * L::kBlk + (kk & 3) * 32) >> 4), idesc_s,
                          kk > 0 ? 1u : 0u);
            mma_commit(s_full + w);
            last_s = ts;
            ++ts;
            key = ts < ntiles ? tile_key(ts) : -1;
            if (key != cur_key) mma_commit(q_empty);  // Qt0 rows no longer needed
            progressed = true;
          }
        }
        if (tp < ts && mbar_test(p_full + (int)(tp & 1), (tp >> 1) & 1)) {
          const int w = (int)(tp & 1), sl = (int)(tp % kSlots);
          tc_fence_after();
          const uint64_t dps = w == 0 ? dp0 : dp1, dkvs = pick3(sl, dkv0, dkv1, dkv2);
#pragma unroll
          for (int kk = 0; kk < L::kKeys / 16; ++kk)
            mma_bf16_ss(tmem + w * 256, dps + (((kk >> 2) * (kRows * 128) + (kk & 3) * 32) >> 4),
                        dkvs + ((kk * 16 * 128) >> 4), idesc_o, kk > 0 ? 1u : 0u);
          mma_commit(o_full + w);
          mma_commit(kv_empty + sl);
          last_o = tp;
          ++tp;
          progressed = true;
        }
        if (progressed) {
          idle_since = global_ns();
        } else if ((__nanosleep(20), *abort_flag)) {
          ok = false;
        } else if (global_ns() - idle_since > kWaitLimitNs) {
          *abort_flag = 1;
          atomicExch(a.status, 1);
          ok = false;
        }
      }
      if (*abort_flag) {
        if (last_s >= 0) drain(s_full + (last_s & 1), (last_s >> 1) & 1);
        if (last_o >= 0) drain(o_full + (last_o & 1), (last_o >> 1) & 1);
      }
    }
    __syncwarp();
  } else {
    // -------------------- softmax + epilogue (two warpgroups) --------------------
    const int w = (warp - 2) >> 2;            // warpgroup 0: warps 2-5, 1: warps 6-9
    const int quad = warp & 3;
    const int r = quad * 32 + lane;           // TMEM lane == tile row
    const int h = PAIR ? (quad >> 1) : 0;     // which sub-item of the tile (warp-uniform)
    const int i = PAIR ? (r & 63) : r;        // position of this row
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t tslot = tmem + w * 256;
    bool ok = true;
    for (long t = w; t < ntiles && ok; t += 2) {
      const long n = s0 + t * H + h;
      const bool have = n < s1;  // warp-uniform
      const KR2Sub sb = kr2_sub(a, have ? n : s0 + t * H);
      const int js = group_start(a.b2, a.c2, sb.q);
      const int nq = group_start(a.b2, a.c2, sb.q + 1) - js;
      int jlo, jhi;
      real_keys(a.real_lo, a.real_hi, a.b2, sb.k, js, nq, &jlo, &jhi);
      ok = mbar_wait(s_full + w, (t >> 1) & 1, abort_flag, a.status);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      float sv[NQ];
#pragma unroll
      for (int c = 0; c < NQ / 16; ++c) {
        float tt[16];
        tmem_ld16(tslot + lane_off + h * NQ + c * 16, tt);
#pragma unroll
        for (int e = 0; e < 16; ++e) sv[c * 16 + e] = tt[e];
      }
      tmem_wait_ld();
      float z, t2;
      r_row_softmax<NQ>(sv, a.sc_log2, jlo, jhi, nq, z, t2);
      // an absent sub-item, or a group without a real key, contributes P = 0
      const float inv = (have && z > 0.f) ? 1.f / z : 0.f;
      uint8_t* pbuf = sP(w);
      // this warp's rows of P were the previous tile's staging: its stores
      // must have read them
      if (lane == 0) bulk_wait_read<0>();
      __syncwarp();
      // P holds R itself (normalised), so [Kt | Y] comes out of the MMA final.
      // Paired tiles: this row's R in its own half of the columns, zeros in
      // the other half.
      auto p_unit = [&](int u) {  // 16-byte unit u (keys 8u .. 8u+7) of this row of P
        return reinterpret_cast<uint4*>(pbuf + (u >> 3) * (kRows * 128) + r * 128 +
                                        (((u & 7) ^ (r & 7)) << 4));
      };
#pragma unroll
      for (int uu = 0; uu < NQ / 8; ++uu) {
        uint4 pk;
        pk.x = pack_bf16x2(sv[8 * uu + 0] * inv, sv[8 * uu + 1] * inv);
        pk.y = pack_bf16x2(sv[8 * uu + 2] * inv, sv[8 * uu + 3] * inv);
        pk.z = pack_bf16x2(sv[8 * uu + 4] * inv, sv[8 * uu + 5] * inv);
        pk.w = pack_bf16x2(sv[8 * uu + 6] * inv, sv[8 * uu + 7] * inv);
        *p_unit(uu + h * (NQ / 8)) = pk;
        if (PAIR) *p_unit(uu + (1 - h) * (NQ / 8)) = make_uint4(0u, 0u, 0u, 0u);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(p_full + w);
      ok = mbar_wait(o_full + w, (t >> 1) & 1, abort_flag, a.status);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const int nblk = (a.write_y ? 2 : 1) * (D / 64);
      const int ycoord = (sb.p * a.b1 + sb.k) * a.c2 + sb.q;
      const bool row_ok = have && i < a.b2;
      const long orow_w = ((((long)sb.g * a.b2 + i) * a.c1 + sb.p) * a.b1 + sb.k) * a.c2 + sb.q;
      // Each warp stores its own 32 rows (positions i0 .. i0 + 31 of its
      // sub-item) through a 4-D box clipped at b2, staging in its own rows
      // of the P buffer (two 4 KB buffers, one per 64-key chunk); a warp
      // whose rows all lie past b2 stores nothing.
      const int i0 = PAIR ? (quad & 1) * 32 : quad * 32;
      const bool store = have && i0 < a.b2;  // warp-uniform
      if (!store) {
        tc_fence_before();
        mbar_arrive(tmem_free + w);
      } else {
        // TMEM loads run one 32-column unit ahead of the staging: unit
        // u + 1 is in flight while unit u is packed into its 64-column
        // block's staging rows; a block goes out once both halves are in.
        float rs[2][32];
        tmem_ld32(tslot + lane_off, rs[0]);
#pragma unroll
        for (int u = 0; u < 4 * (D / 64); ++u) {
          if (u < 2 * nblk) {
            const int cb = u >> 1, hf = u & 1;
            tmem_wait_ld();  // unit u is in registers
            if (u == 2 * nblk - 1) {  // slot fully read out: the MMA may reuse it
              tc_fence_before();
              mbar_arrive(tmem_free + w);
            } else {
              tmem_ld32(tslot + lane_off + (u + 1) * 32, rs[(u + 1) & 1]);
            }
            uint8_t* buf = pbuf + (cb & 1) * (kRows * 128) + quad * 32 * 128;
            if (hf == 0) {
              if (cb >= 2 && lane == 0) bulk_wait_read<1>();  // store of block cb-2 has read buf
              __syncwarp();
            }
#pragma unroll
            for (int uu = 0; uu < 4; ++uu) {
              const float* v = rs[u & 1] + 8 * uu;
              uint4 pk;
              pk.x = pack_bf16x2(v[0], v[1]);
              pk.y = pack_bf16x2(v[2], v[3]);
              pk.z = pack_bf16x2(v[4], v[5]);
              pk.w = pack_bf16x2(v[6], v[7]);
              const int chunk = hf * 4 + uu;
              *reinterpret_cast<uint4*>(buf + lane * 128 + ((chunk ^ (lane & 7)) << 4)) = pk;
            }
            if (hf == 1) {
              fence_proxy_async_smem();
              __syncwarp();
              if (lane == 0) {
                tma_store_4d(cb < D / 64 ? &tm_kt : &tm_y, buf, (cb % (D / 64)) * 64, ycoord,
                             i0, sb.g);
                bulk_commit();
              }
            }
          }
        }
      }
      if (row_ok) a.hs[orow_w] = z > 0.f ? logf(z) - t2 * 0.69314718055994531f / z : -INFINITY;
    }
    if (lane == 0) bulk_wait<0>();  // stores done reading shared memory before exit
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// Non-final L-update on the tensor cores, for rows of at most 128 keys
// (nk = b1 c2) and row groups of at most 128 rows.  One CTA of eight warps
// per (g, i, p):
//   S = q Kt^T / sqrt(d) + Hs           128 rows x 128 keys in TMEM
//   L = softmax over the valid keys      exact, two threads per row (64 keys
//                                        each; maximum and sum combined in
//                                        shared memory); rows past the group
//                                        and pad rows get L = 0
//   [Qt~ | c] = L^T [Q | 1]               128 keys x (d + 64) in TMEM, over the
//                                        columns S held; c = column sums of L
//   Qt_{k,p,q,i} = Qt~ / c (0 if c = 0)   thread = key (warps 0-3), bf16 rows
// (MonarchAttention OpenReview discussion, the alternating maximisation: the
// L-update's row softmax, then the aggregated queries of the next
// R-update.)  L goes to shared memory as bf16 in [row][key] order: with keys
// as the M dimension that is the MN-major A operand of the second product.
// Q, staged K-major for the first product, is read again as its MN-major B
// operand (d contiguous per row), with a constant 64-column block of ones
// appended, whose products are the column sums.
// ---------------------------------------------------------------------------
template <int D>
struct KLLayout {
  static constexpr int kChunk = kRows * 128;              // 128 rows x 64 bf16, swizzled
  static constexpr int kQOff = 0;                          // D / 64 chunks, then the ones
  static constexpr int kOnesOff = D / 64 * kChunk;
  static constexpr int kKtOff = kOnesOff + kChunk;         // D / 64 chunks of 128 keys
  static constexpr int kPOff = kKtOff + D / 64 * kChunk;   // keys 0-63, keys 64-127
  static constexpr int kBiasOff = kPOff + 2 * kChunk;      // float [128]
  static constexpr int kBarOff = kBiasOff + 128 * 4;
  static constexpr int kBytes = kBarOff + 8 * 8;
  static constexpr uint32_t kTmemCols = 256;
  static_assert(D == 64 || D == 128, "head dimension");
};

struct KLArgs {
  const float* hs;  // [G][b2][c1][nk]
  bf16* qt;         // [G][b1 k][c1 p][c2 q][b2 i][d]
  int b1, b2, c1, c2, nk, real_lo, real_hi;
  float sc;
  int* status;
  int tr;  // token order of q (see Problem)
};

template <int D>
__global__ void __launch_bounds__(256)
    kl_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kt,
              KLArgs a) {
  using L = KLLayout<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5;
  if (smem_u32(smem) & 1023u) {
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
  uint8_t* sOnes = smem + L::kOnesOff;
  uint8_t* sKt = smem + L::kKtOff;
  uint8_t* sP = smem + L::kPOff;
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
  // the ones block: bf16 1.0 in every element
  for (int x = tid; x < L::kChunk / 16; x += 256)
    reinterpret_cast<uint4*>(sOnes)[x] = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u,
                                                     0x3F803F80u);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;  // warp w: lanes of w % 4
  pdl_wait();  // Kt and the entropies come from the previous kernel
  pdl_launch_dependents();
  bool issued_s = false, issued_o = false;
  if (tid == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_kt);
    mbar_arrive_expect_tx(load_full, 2 * (D / 64) * L::kChunk);
    const int2 qyz = q_slab_yz(a.tr, g, a.b1, a.b2, i, l0);
#pragma unroll
    for (int c = 0; c < D / 64; ++c) {
      tma_load_3d(sQ + c * L::kChunk, &tm_q, load_full, c * 64, qyz.x, qyz.y);
      tma_load_2d(sKt + c * L::kChunk, &tm_kt, load_full, c * 64, (int)key_row0);
    }
  }
  if (tid < 128) sBias[tid] = tid < a.nk ? a.hs[key_row0 + tid] : -INFINITY;
  __syncthreads();
  if (tid == 0 && mbar_wait(load_full, 0, abort_flag, a.status)) {
    tc_fence_after();
    const uint64_t dq = desc_kmajor(smem_u32(sQ)), dk = desc_kmajor(smem_u32(sKt));
    const uint32_t idesc = idesc_bf16(kRows, 128, false);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk)
      mma_bf16_ss(tmem, dq + (((kk >> 2) * L::kChunk + (kk & 3) * 32) >> 4),
                  dk + (((kk >> 2) * L::kChunk + (kk & 3) * 32) >> 4), idesc, kk > 0 ? 1u : 0u);
    mma_commit(s_full);
    issued_s = true;
  }
  // ---- softmax: two threads per row r of the group (warps w and w + 4
  // share the TMEM lanes), each over 64 keys; the row's maximum and sum are
  // combined through the Kt buffer, dead once S is complete ----
  const int r = tid & 127, half = tid >> 7, l = l0 + r;
  const bool row_real = l < l1 && l * a.b2 + i >= a.real_lo && l * a.b2 + i < a.real_hi;
  float* red = reinterpret_cast<float*>(sKt);  // [max: 2][128], [sum: 2][128]
  bool ok = mbar_wait(s_full, 0, abort_flag, a.status);
  ok = __syncthreads_and(ok);
  float sv[64];
  if (ok) {
    tc_fence_after();
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      float t[32];
      tmem_ld32(tmem + lane_off + half * 64 + c * 32, t);
#pragma unroll
      for (int e = 0; e < 32; ++e) sv[c * 32 + e] = t[e];
    }
    tmem_wait_ld();
    // logits (-inf past nk and for groups without a real key) and maxima
    float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
    const float2 sc2 = make_float2(a.sc, a.sc);
#pragma unroll
    for (int c = 0; c < 64; c += 4) {
      const float4 b4 = *reinterpret_cast<const float4*>(sBias + half * 64 + c);
      const float2 lo = fma2(make_float2(sv[c], sv[c + 1]), sc2, make_float2(b4.x, b4.y));
      const float2 hi = fma2(make_float2(sv[c + 2], sv[c + 3]), sc2, make_float2(b4.z, b4.w));
      sv[c] = lo.x;
      sv[c + 1] = lo.y;
      sv[c + 2] = hi.x;
      sv[c + 3] = hi.y;
      const int mm = (c >> 2) & 1;
      mx[mm] = max3(mx[mm], lo.x, lo.y);
      mx[2 + mm] = max3(mx[2 + mm], hi.x, hi.y);
    }
    red[half * 128 + r] = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
  }
  ok = __syncthreads_and(ok);
  float m = 0.f;
  if (ok) {
    m = fmaxf(red[r], red[128 + r]);
    if (m == -INFINITY) m = 0.f;
    const float2 l2e = make_float2(kLog2e, kLog2e), nm2 = make_float2(-m * kLog2e, -m * kLog2e);
    float2 z01 = make_float2(0.f, 0.f), z23 = z01;
#pragma unroll
    for (int c = 0; c < 64; c += 4) {
      const float2 x0 = fma2(make_float2(sv[c], sv[c + 1]), l2e, nm2);
      const float2 x1 = fma2(make_float2(sv[c + 2], sv[c + 3]), l2e, nm2);
      sv[c] = ex2(x0.x);
      sv[c + 1] = ex2(x0.y);
      sv[c + 2] = ex2(x1.x);
      sv[c + 3] = ex2(x1.y);
      z01 = add2(z01, make_float2(sv[c], sv[c + 1]));
      z23 = add2(z23, make_float2(sv[c + 2], sv[c + 3]));
    }
    red[256 + half * 128 + r] = (z01.x + z01.y) + (z23.x + z23.y);
  }
  ok = __syncthreads_and(ok);
  if (ok) {
    const float z = red[256 + r] + red[384 + r];
    const float inv = (row_real && z > 0.f) ? 1.f / z : 0.f;
#pragma unroll
    for (int uu = 0; uu < 8; ++uu) {  // this half's 16-byte units (keys 8u .. 8u + 7)
      uint4 pk;
      pk.x = pack_bf16x2(sv[8 * uu + 0] * inv, sv[8 * uu + 1] * inv);
      pk.y = pack_bf16x2(sv[8 * uu + 2] * inv, sv[8 * uu + 3] * inv);
      pk.z = pack_bf16x2(sv[8 * uu + 4] * inv, sv[8 * uu + 5] * inv);
      pk.w = pack_bf16x2(sv[8 * uu + 6] * inv, sv[8 * uu + 7] * inv);
      *reinterpret_cast<uint4*>(sP + half * L::kChunk + r * 128 + ((uu ^ (r & 7)) << 4)) = pk;
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  ok = __syncthreads_and(ok);
  if (ok && tid == 0) {
    tc_fence_after();
    // keys x (d + 64) over the 128 rows, 16 rows per instruction
    const uint64_t dp = desc_mnmajor(smem_u32(sP), L::kChunk);
    const uint64_t dq = desc_mnmajor(smem_u32(sQ), L::kChunk);
    const uint32_t idesc = idesc_bf16(kRows, D + 64, true, true);
#pragma unroll
    for (int kk = 0; kk < kRows / 16; ++kk)
      mma_bf16_ss(tmem, dp + ((kk * 16 * 128) >> 4), dq + ((kk * 16 * 128) >> 4), idesc,
                  kk > 0 ? 1u : 0u);
    mma_commit(o_full);
    issued_o = true;
  }
  // ---- epilogue, thread = key m = k c2 + q ----
  if (ok) ok = mbar_wait(o_full, 0, abort_flag, a.status);
  ok = __syncthreads_and(ok);
  if (ok && warp < 4) {
    tc_fence_after();
    const int m = tid;
    float cs[32];
    tmem_ld32(tmem + lane_off + D, cs);
    tmem_wait_ld();
    const float invc = cs[0] > 0.f ? 1.f / cs[0] : 0.f;
    const int k = m / a.c2, q = m % a.c2;
    bf16* dst = a.qt + (((((long)g * a.b1 + k) * a.c1 + p) * a.c2 + q) * a.b2 + i) * D;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      float t[32];
      tmem_ld32(tmem + lane_off + c * 32, t);
      tmem_wait_ld();
      if (m < a.nk) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          uint4 pk;
          pk.x = pack_bf16x2(t[8 * u + 0] * invc, t[8 * u + 1] * invc);
          pk.y = pack_bf16x2(t[8 * u + 2] * invc, t[8 * u + 3] * invc);
          pk.z = pack_bf16x2(t[8 * u + 4] * invc, t[8 * u + 5] * invc);
          pk.w = pack_bf16x2(t[8 * u + 6] * invc, t[8 * u + 7] * invc);
          *reinterpret_cast<uint4*>(dst + c * 32 + 8 * u) = pk;
        }
      }
    }
  }
  if (tid == 0 && *abort_flag) {  // drain what this CTA issued (bounded)
    if (!issued_s) drain(load_full, 0);
    if (issued_s) drain(s_full, 0);
    if (issued_o) drain(o_full, 0);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Non-final L-update for L rows of more than 128 keys or row groups of more
// than 128 rows, in two passes.
//
// kls_kernel, one CTA per (g, i, p, row tile): the log-sum-exp of every row
// over all b1 c2 keys, S = q Kt^T / sqrt(d) + Hs a 128-key tile at a time
// (double-buffered in TMEM), running max and sum in registers, one row per
// thread of warps 1-4; warp 0 loads (TMA) and issues the MMAs.  No barrier
// joins the row warps: each stages the tile's biases in its own shared
// copy (coalesced loads issued before it waits for S, then broadcasts), so
// a warp whose bounded wait gives up cannot leave the others waiting.
//
// klm_kernel, one CTA per (g, i, p, key tile): for every row tile, S again,
// P = exp(S - lse) (rows past the group and pad rows 0), and
// [Qt~ | c] += P^T [Q | 1] in TMEM across the row tiles (the product of
// kl_kernel, accumulated); then thread = key writes Qt = Qt~ / c.  Queries
// and P are double-buffered: the next row tile's queries load, and the
// aggregation of this one runs, while the next S and softmax proceed.
// ---------------------------------------------------------------------------
template <int D>
struct KLSLayout {
  static constexpr int kChunk = kRows * 128;
  static constexpr int kQOff = 0;                            // D / 64 chunks
  static constexpr int kKtOff = D / 64 * kChunk;             // 2 slots of D / 64 chunks
  static constexpr int kBiasOff = kKtOff + 2 * (D / 64) * kChunk;  // float [4 row warps][128]
  static constexpr int kBarOff = kBiasOff + 4 * 128 * 4;
  static constexpr int kBytes = kBarOff + 16 * 8;
};

struct KLSArgs {
  const float* hs;  // [G][b2][c1][nk]
  float* lse;       // [G][b2][b1]
  int b1, b2, c1, nk, row_tiles, real_lo, real_hi;
  float sc;
  int* status;
  int tr;  // token order of q (see Problem)
};

template <int D>
__global__ void __launch_bounds__(160)
    kls_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kt,
               KLSArgs a) {
  using L = KLSLayout<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (smem_u32(smem) & 1023u) {
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
  const long key_row0 = ((long)(g * a.b2 + i) * a.c1 + p) * a.nk;
  const int n_kt = (a.nk + 127) / 128;
  uint8_t* sQ = smem + L::kQOff;
  auto sKt = [&](int sl) { return smem + L::kKtOff + sl * (D / 64) * L::kChunk; };
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* q_full = bars + 0;
  uint64_t* kt_full = bars + 1;   // [2]
  uint64_t* kt_empty = bars + 3;  // [2]
  uint64_t* s_full = bars + 5;    // [2]
  uint64_t* s_free = bars + 7;    // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 9);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 10);
  if (tid == 0) {
    mbar_init(q_full, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(kt_full + b, 1);
      mbar_init(kt_empty + b, 1);
      mbar_init(s_full + b, 1);
      mbar_init(s_free + b, 128);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();  // Kt and the entropies come from the previous kernel
  pdl_launch_dependents();
  if (warp == 0) {
    // ---- loads and MMAs, one thread ----
    if (lane == 0) {
      bool ok = true;
      long loaded = 0, issued = 0;
      mbar_arrive_expect_tx(q_full, (D / 64) * L::kChunk);
      const int2 qyz = q_slab_yz(a.tr, g, a.b1, a.b2, i, row0);
#pragma unroll
      for (int c = 0; c < D / 64; ++c)
        tma_load_3d(sQ + c * L::kChunk, &tm_q, q_full, c * 64, qyz.x, qyz.y);
      auto load_kt = [&](int kt) {
        const int sl = kt & 1;
        mbar_arrive_expect_tx(kt_full + sl, (D / 64) * L::kChunk);
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          tma_load_2d(sKt(sl) + c * L::kChunk, &tm_kt, kt_full + sl, c * 64,
                      (int)(key_row0 + kt * 128));
      };
      for (; loaded < 2 && loaded < n_kt; ++loaded) load_kt((int)loaded);
      ok = mbar_wait(q_full, 0, abort_flag, a.status);
      const uint32_t idesc = idesc_bf16(kRows, 128, false);
      for (int kt = 0; kt < n_kt && ok; ++kt) {
        const int sl = kt & 1;
        ok = mbar_wait(kt_full + sl, (kt >> 1) & 1, abort_flag, a.status) &&
             (kt < 2 || mbar_wait(s_free + sl, ((kt >> 1) - 1) & 1, abort_flag, a.status));
        if (!ok) break;
        tc_fence_after();
        const uint64_t dq = desc_kmajor(smem_u32(sQ)), dk = desc_kmajor(smem_u32(sKt(sl)));
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_bf16_ss(tmem + sl * 128, dq + (((kk >> 2) * L::kChunk + (kk & 3) * 32) >> 4),
                      dk + (((kk >> 2) * L::kChunk + (kk & 3) * 32) >> 4), idesc,
                      kk > 0 ? 1u : 0u);
        mma_commit(s_full + sl);
        mma_commit(kt_empty + sl);
        issued = kt + 1;
        if (loaded < n_kt) {
          ok = mbar_wait(kt_empty + sl, (kt >> 1) & 1, abort_flag, a.status);
          if (ok) load_kt((int)loaded++);
        }
      }
      if (*abort_flag) {
        drain(q_full, 0);
        for (long t = loaded >= 2 ? loaded - 2 : 0; t < loaded; ++t)
          drain(kt_full + (t & 1), (t >> 1) & 1);
        if (issued > 0) drain(s_full + ((issued - 1) & 1), ((issued - 1) >> 1) & 1);
      }
    }
    __syncwarp();
  } else {
    // ---- row statistics, thread = row ----
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const int l = row0 + r;
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    float m_run = -INFINITY, z = 0.f;
    float* wbias = reinterpret_cast<float*>(smem + L::kBiasOff) + (warp - 1) * 128;
    bool ok = true;
    for (int kt = 0; kt < n_kt && ok; ++kt) {
      const int sl = kt & 1;
      const int col0 = kt * 128;
      // this tile's entropy biases, -inf past the row's keys (which also
      // masks the zero-filled Kt rows there)
      {
        const float* hs_t = a.hs + key_row0 + col0;
        float b[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
          b[e] = col0 + e * 32 + lane < a.nk ? __ldg(hs_t + e * 32 + lane) : -INFINITY;
        __syncwarp();  // the previous tile's reads of wbias are done
#pragma unroll
        for (int e = 0; e < 4; ++e) wbias[e * 32 + lane] = b[e];
        __syncwarp();
      }
      ok = mbar_wait(s_full + sl, (kt >> 1) & 1, abort_flag, a.status);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      float sv[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float t[32];
        tmem_ld32(tmem + sl * 128 + lane_off + c * 32, t);
#pragma unroll
        for (int e = 0; e < 32; ++e) sv[c * 32 + e] = t[e];
      }
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(s_free + sl);
      // logits, maxima and sums on packed pairs (scalar roundings); the
      // partial sums over columns c mod 4 are the pairs (0, 1) and (2, 3)
      float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
      const float2 sc2 = make_float2(a.sc, a.sc);
#pragma unroll
      for (int c = 0; c < 128; c += 4) {
        const float4 b4 = *reinterpret_cast<const float4*>(wbias + c);
        const float2 lo = fma2(make_float2(sv[c], sv[c + 1]), sc2, make_float2(b4.x, b4.y));
        const float2 hi = fma2(make_float2(sv[c + 2], sv[c + 3]), sc2, make_float2(b4.z, b4.w));
        sv[c] = lo.x;
        sv[c + 1] = lo.y;
        sv[c + 2] = hi.x;
        sv[c + 3] = hi.y;
        const int m = (c >> 2) & 1;
        mx[m] = max3(mx[m], lo.x, lo.y);
        mx[2 + m] = max3(mx[2 + m], hi.x, hi.y);
      }
      const float mt = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
      const float mn = fmaxf(m_run, mt);
      const float base = mn > -INFINITY ? mn : 0.f;
      const float2 nb = make_float2(-base, -base), l2e = make_float2(kLog2e, kLog2e);
      float2 z01 = make_float2(0.f, 0.f), z23 = z01;
#pragma unroll
      for (int c = 0; c < 128; c += 4) {
        const float2 x0 = mul2(add2(make_float2(sv[c], sv[c + 1]), nb), l2e);
        const float2 x1 = mul2(add2(make_float2(sv[c + 2], sv[c + 3]), nb), l2e);
        z01 = add2(z01, make_float2(ex2(x0.x), ex2(x0.y)));
        z23 = add2(z23, make_float2(ex2(x1.x), ex2(x1.y)));
      }
      z = z * (m_run > -INFINITY ? ex2((m_run - base) * kLog2e) : 0.f) +
          ((z01.x + z01.y) + (z23.x + z23.y));
      m_run = mn;
    }
    if (ok && l < l1) a.lse[((long)g * a.b2 + i) * a.b1 + l] = m_run + logf(z);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

template <int D>
struct KLMLayout {
  static constexpr int kChunk = kRows * 128;
  // two query buffers, each D / 64 chunks and then a chunk of ones (the
  // [Q | 1] operand), so that the next row tile's queries load during this one
  static constexpr int kQBufBytes = (D / 64 + 1) * kChunk;
  static constexpr int kQOff = 0;
  static constexpr int kKtOff = 2 * kQBufBytes;            // D / 64 chunks of 128 keys
  static constexpr int kPOff = kKtOff + D / 64 * kChunk;   // 2 buffers: keys 0-63, 64-127
  static constexpr int kBiasOff = kPOff + 4 * kChunk;      // float [128]
  static constexpr int kBarOff = kBiasOff + 128 * 4;
  static constexpr int kBytes = kBarOff + 10 * 8;
  static constexpr uint32_t kTmemCols = D + 64 + 128 <= 256 ? 256 : 512;
  static constexpr uint32_t kSCol = kTmemCols - 128;       // S; [Qt~ | c] at [0, D + 64)
  static_assert(kBytes <= 227 * 1024, "shared memory");
};

struct KLMArgs {
  const float* hs;   // [G][b2][c1][nk]
  const float* lse;  // [G][b2][b1]
  bf16* qt;          // [G][b1 k][c1 p][c2 q][b2 i][d]
  int b1, b2, c1, c2, nk, key_tiles, real_lo, real_hi;
  float sc;
  int* status;
  int tr;  // token order of q (see Problem)
};

template <int D>
__global__ void __launch_bounds__(256)
    klm_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kt,
               KLMArgs a) {
  using L = KLMLayout<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5;
  if (smem_u32(smem) & 1023u) {
    if (tid == 0) atomicExch(a.status, 2);
    return;
  }
  int bid = blockIdx.x;
  const int kt = bid % a.key_tiles;
  bid /= a.key_tiles;
  const int p = bid % a.c1;
  bid /= a.c1;
  const int i = bid % a.b2;
  const int g = bid / a.b2;
  const int l0 = group_start(a.b1, a.c1, p), l1 = group_start(a.b1, a.c1, p + 1);
  const long key_row0 = ((long)(g * a.b2 + i) * a.c1 + p) * a.nk + kt * 128;
  const int n_rt = (l1 - l0 + kRows - 1) / kRows;
  auto sQ = [&](int b) { return smem + L::kQOff + b * L::kQBufBytes; };
  uint8_t* sKt = smem + L::kKtOff;
  auto sP = [&](int b) { return smem + L::kPOff + b * 2 * L::kChunk; };
  float* sBias = reinterpret_cast<float*>(smem + L::kBiasOff);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* kt_full = bars + 0;
  uint64_t* q_full = bars + 1;  // [2], one per query buffer
  uint64_t* s_full = bars + 3;
  uint64_t* o_full = bars + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 6);
  if (tid == 0) {
    mbar_init(kt_full, 1);
    mbar_init(q_full, 1);
    mbar_init(q_full + 1, 1);
    mbar_init(s_full, 1);
    mbar_init(o_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
  }
  for (int b = 0; b < 2; ++b) {
    uint4* ones = reinterpret_cast<uint4*>(sQ(b) + D / 64 * L::kChunk);
    for (int x = tid; x < L::kChunk / 16; x += 256)
      ones[x] = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tmem_s = tmem + L::kSCol;
  const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;  // warp w: lanes of w % 4
  pdl_wait();  // Kt, the entropies and the row statistics come from earlier kernels
  pdl_launch_dependents();
  auto load_q = [&](int rt) {  // row tile rt's queries into buffer rt & 1 (one thread)
    const int b = rt & 1;
    mbar_arrive_expect_tx(q_full + b, (D / 64) * L::kChunk);
    const int2 qyz = q_slab_yz(a.tr, g, a.b1, a.b2, i, l0 + rt * kRows);
#pragma unroll
    for (int c = 0; c < D / 64; ++c)
      tma_load_3d(sQ(b) + c * L::kChunk, &tm_q, q_full + b, c * 64, qyz.x, qyz.y);
  };
  int q_loads = 0;
  if (tid == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_kt);
    mbar_arrive_expect_tx(kt_full, (D / 64) * L::kChunk);
#pragma unroll
    for (int c = 0; c < D / 64; ++c)
      tma_load_2d(sKt + c * L::kChunk, &tm_kt, kt_full, c * 64, (int)key_row0);
    load_q(0);
    q_loads = 1;
  }
  const int key = kt * 128 + (tid & 127);
  if (tid < 128) sBias[tid] = key < a.nk ? a.hs[key_row0 + tid] : -INFINITY;
  __syncthreads();
  const float* lse_i = a.lse + ((long)g * a.b2 + i) * a.b1;
  bool ok = true;
  int issued_s = 0, issued_o = 0;
  for (int rt = 0; rt < n_rt && ok; ++rt) {
    const int row0 = l0 + rt * kRows;
    const int qb = rt & 1;
    if (tid == 0) {
      // the next row tile's queries go to the other buffer once the
      // aggregation that read it (row tile rt - 1) is done
      if (rt + 1 < n_rt) {
        if (rt >= 1) ok = mbar_wait(o_full, (rt - 1) & 1, abort_flag, a.status);
        if (ok) {
          load_q(rt + 1);
          ++q_loads;
        }
      }
      ok = ok && mbar_wait(q_full + qb, (rt >> 1) & 1, abort_flag, a.status) &&
           (rt > 0 || mbar_wait(kt_full, 0, abort_flag, a.status));
      if (ok) {
        tc_fence_after();
        const uint64_t dq = desc_kmajor(smem_u32(sQ(qb))), dk = desc_kmajor(smem_u32(sKt));
        const uint32_t idesc = idesc_bf16(kRows, 128, false);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_bf16_ss(tmem_s, dq + (((kk >> 2) * L::kChunk + (kk & 3) * 32) >> 4),
                      dk + (((kk >> 2) * L::kChunk + (kk & 3) * 32) >> 4), idesc,
                      kk > 0 ? 1u : 0u);
        mma_commit(s_full);
        ++issued_s;
      }
    }
    // ---- P = exp(S - lse): two threads per row (warps w and w + 4 share the
    // TMEM lanes), each over 64 of the tile's keys ----
    const int r = tid & 127, half = tid >> 7, l = row0 + r;
    const bool row_real = l < l1 && l * a.b2 + i >= a.real_lo && l * a.b2 + i < a.real_hi;
    const float lse_row = row_real ? lse_i[l] : 0.f;
    ok = ok && mbar_wait(s_full, rt & 1, abort_flag, a.status);
    ok = __syncthreads_and(ok);
    if (!ok) break;
    tc_fence_after();
    float sv[64];
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      float t[32];
      tmem_ld32(tmem_s + lane_off + half * 64 + c * 32, t);
#pragma unroll
      for (int e = 0; e < 32; ++e) sv[c * 32 + e] = t[e];
    }
    tmem_wait_ld();
    // P of this row tile into buffer rt & 1, last read by the aggregation of
    // row tile rt - 2 (complete: its successor's was waited for above)
    uint8_t* pbuf = sP(rt & 1);
#pragma unroll
    for (int uu = 0; uu < 8; ++uu) {  // 16-byte unit u holds keys 8u .. 8u + 7
      const int u = half * 8 + uu;
      float w[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float x = fmaf(sv[8 * uu + e], a.sc, sBias[8 * u + e]);
        w[e] = row_real && x > -INFINITY ? ex2((x - lse_row) * kLog2e) : 0.f;
      }
      uint4 pk;
      pk.x = pack_bf16x2(w[0], w[1]);
      pk.y = pack_bf16x2(w[2], w[3]);
      pk.z = pack_bf16x2(w[4], w[5]);
      pk.w = pack_bf16x2(w[6], w[7]);
      *reinterpret_cast<uint4*>(pbuf + half * L::kChunk + r * 128 + ((uu ^ (r & 7)) << 4)) = pk;
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      const uint64_t dp = desc_mnmajor(smem_u32(pbuf), L::kChunk);
      const uint64_t dq = desc_mnmajor(smem_u32(sQ(qb)), L::kChunk);
      const uint32_t idesc = idesc_bf16(kRows, D + 64, true, true);
#pragma unroll
      for (int kk = 0; kk < kRows / 16; ++kk)
        mma_bf16_ss(tmem, dp + ((kk * 16 * 128) >> 4), dq + ((kk * 16 * 128) >> 4), idesc,
                    (rt > 0 || kk > 0) ? 1u : 0u);
      mma_commit(o_full);
      ++issued_o;
    }
  }
  // the last aggregation complete: [Qt~ | c] final
  if (tid == 0 && ok && issued_o > 0)
    ok = mbar_wait(o_full, (issued_o - 1) & 1, abort_flag, a.status);
  ok = __syncthreads_and(ok);
  // ---- epilogue, thread = key (warps 0-3) ----
  if (ok && warp < 4) {
    tc_fence_after();
    float cs[32];
    tmem_ld32(tmem + lane_off + D, cs);
    tmem_wait_ld();
    const float invc = cs[0] > 0.f ? 1.f / cs[0] : 0.f;
    const int kk_ = key / a.c2, q = key % a.c2;
    bf16* dst = a.qt + (((((long)g * a.b1 + kk_) * a.c1 + p) * a.c2 + q) * a.b2 + i) * D;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      float t[32];
      tmem_ld32(tmem + lane_off + c * 32, t);
      tmem_wait_ld();
      if (key < a.nk) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          uint4 pk;
          pk.x = pack_bf16x2(t[8 * u + 0] * invc, t[8 * u + 1] * invc);
          pk.y = pack_bf16x2(t[8 * u + 2] * invc, t[8 * u + 3] * invc);
          pk.z = pack_bf16x2(t[8 * u + 4] * invc, t[8 * u + 5] * invc);
          pk.w = pack_bf16x2(t[8 * u + 6] * invc, t[8 * u + 7] * invc);
          *reinterpret_cast<uint4*>(dst + c * 32 + 8 * u) = pk;
        }
      }
    }
  }
  if (tid == 0 && *abort_flag) {  // drain what this CTA issued (bounded)
    drain(kt_full, 0);
    for (int t = q_loads >= 2 ? q_loads - 2 : 0; t < q_loads; ++t) drain(q_full + (t & 1), (t >> 1) & 1);
    if (issued_s > 0) drain(s_full, (issued_s - 1) & 1);
    if (issued_o > 0) drain(o_full, (issued_o - 1) & 1);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Self-test of the bounded-wait path: one CTA waits on an mbarrier that
// nothing ever arrives on, gives up after limit_ns, records the timeout in
// the status word and returns normally.
// ---------------------------------------------------------------------------
__global__ void selftest_timeout_kernel(int* status, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_word;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_word = 0;
    fence_mbar_init();
  }
  __syncthreads();
  (void)mbar_wait(&bar, 0, &abort_word, status, limit_ns);
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
// strides in bytes for dims 1.. .  A map is a pure function of its
// arguments, so encoded maps are kept in a small cache: repeated calls on the
// same buffers skip the host-side encoding.
struct MapKey {
  const void* base;
  int rank;
  cuuint64_t dims[4], str[3];
  cuuint32_t box[4];
  bool operator==(const MapKey& o) const {
    if (base != o.base || rank != o.rank) return false;
    for (int i = 0; i < rank; ++i)
      if (dims[i] != o.dims[i] || box[i] != o.box[i]) return false;
    for (int i = 0; i + 1 < rank; ++i)
      if (str[i] != o.str[i]) return false;
    return true;
  }
};

bool make_map(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims,
              const cuuint64_t* strides, const cuuint32_t* box) {
  static std::mutex mu;
  static MapKey keys[64];
  static CUtensorMap maps[64];
  static int used = 0, next = 0;
  if (rank < 1 || rank > 4) return false;
  MapKey key = {};
  key.base = base;
  key.rank = rank;
  for (int i = 0; i < rank; ++i) {
    key.dims[i] = dims[i];
    key.box[i] = box[i];
  }
  for (int i = 0; i + 1 < rank; ++i) key.str[i] = strides[i];
  {
    std::lock_guard<std::mutex> lock(mu);
    for (int e = 0; e < used; ++e)
      if (keys[e] == key) {
        *m = maps[e];
        return true;
      }
  }
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  if (fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides, box,
         estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  std::lock_guard<std::mutex> lock(mu);
  keys[next] = key;
  maps[next] = *m;
  next = (next + 1) % 64;
  if (used < 64) ++used;
  return true;
}

// 3-D map of q whose box is the 128 rows l (from row0) of one position i:
// Monarch order (rows l are b2*d apart) or its transpose (rows l adjacent).
bool make_q_slab_map(CUtensorMap* m, const bf16* q, const Problem& pb, int D) {
  if (pb.tr) {
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)pb.b1, (cuuint64_t)pb.G * pb.b2};
    const cuuint64_t str[2] = {(cuuint64_t)D * 2, (cuuint64_t)pb.b1 * D * 2};
    const cuuint32_t box[3] = {64, kRows, 1};
    return make_map(m, q, 3, dims, str, box);
  }
  const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)pb.b2, (cuuint64_t)pb.G * pb.b1};
  const cuuint64_t str[2] = {(cuuint64_t)D * 2, (cuuint64_t)pb.b2 * D * 2};
  const cuuint32_t box[3] = {64, 1, kRows};
  return make_map(m, q, 3, dims, str, box);
}

// 3-D map of k or v whose box is `rows` keys j (from j0) of one chunk k: rows
// j adjacent (Monarch order) or b1*d apart (transposed); rows past b2 read as
// zeros.
bool make_kv_map(CUtensorMap* m, const bf16* x, const Problem& pb, int D, int rows) {
  if (pb.tr) {
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)pb.b1, (cuuint64_t)pb.G * pb.b2};
    const cuuint64_t str[2] = {(cuuint64_t)D * 2, (cuuint64_t)pb.b1 * D * 2};
    const cuuint32_t box[3] = {64, 1, (cuuint32_t)rows};
    return make_map(m, x, 3, dims, str, box);
  }
  const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)pb.b2, (cuuint64_t)pb.G * pb.b1};
  const cuuint64_t str[2] = {(cuuint64_t)D * 2, (cuuint64_t)pb.b2 * D * 2};
  const cuuint32_t box[3] = {64, (cuuint32_t)rows, 1};
  return make_map(m, x, 3, dims, str, box);
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
    if (attr_err == cudaSuccess)
      attr_err = cudaFuncSetAttribute(ko_kernel<D, NK>,
                                      cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  });
  if (attr_err != cudaSuccess) return attr_err;
  const int nk = pb.b1 * pb.c2;
  const long key_rows = (long)pb.G * pb.b2 * pb.c1 * nk;
  CUtensorMap tq, tk, tyv;
  {
    if (!make_q_slab_map(&tq, q, pb, D)) return cudaErrorInvalidValue;
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
  const long items = (long)pb.G * pb.b2 * pb.c1 * a.row_tiles;
  if (items >= (1L << 31)) return cudaErrorInvalidValue;
  a.n_items = (int)items;
  a.sc = pb.sc;
  a.status = status;
  a.tr = pb.tr;
  const int grid = (int)std::min<long>(items, 2L * num_sms());
  return timed_launch("tc_l_output", stream, launches, [&] {
    return launch_pdl(ko_kernel<D, NK>, dim3(grid), dim3(192), L::kAlloc, stream, tq, tk, tyv, a);
  });
}

template <int D, int NK>
cudaError_t launch_ko1(const bf16* q, const bf16* kt, const bf16* y, const float* hs, bf16* out,
                       const Problem& pb, int* status, cudaStream_t stream, int* launches) {
  using L = KO1Layout<D, NK>;
  static std::once_flag attr_once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(attr_once, [] {
    attr_err = cudaFuncSetAttribute(ko1_kernel<D, NK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    L::kAlloc);
    if (attr_err == cudaSuccess)
      attr_err = cudaFuncSetAttribute(ko1_kernel<D, NK>,
                                      cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  });
  if (attr_err != cudaSuccess) return attr_err;
  const int nk = pb.b1 * pb.c2;
  if (nk > NK) return cudaErrorInvalidValue;
  const long key_rows = (long)pb.G * pb.b2 * pb.c1 * nk;
  CUtensorMap tq, tk, tyv;
  {
    if (!make_q_slab_map(&tq, q, pb, D)) return cudaErrorInvalidValue;
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
  const long items = (long)pb.G * pb.b2 * pb.c1 * a.row_tiles;
  if (items >= (1L << 31)) return cudaErrorInvalidValue;
  a.n_items = (int)items;
  a.sc = pb.sc;
  a.status = status;
  a.tr = pb.tr;
  const int grid = (int)std::min<long>(items, 2L * num_sms());
  return timed_launch("tc_l_output", stream, launches, [&] {
    return launch_pdl(ko1_kernel<D, NK>, dim3(grid), dim3(192), L::kAlloc, stream, tq, tk, tyv, a);
  });
}

// Output kernel by key count: one warp per (g, i, p) on the CUDA cores for
// rows of <= 8 keys, one key tile per row when b1*c2 <= 64, else the
// online-softmax kernel over 64-key tiles.
template <int D>
cudaError_t dispatch_ko(const bf16* q, const bf16* kt, const bf16* y, const float* hs, bf16* out,
                        const Problem& pb, int* status, cudaStream_t stream, int* launches) {
  const int nk = pb.b1 * pb.c2;
  if (small_out_fits(pb)) return launch_small_out(q, kt, y, hs, out, pb, stream, launches);
  if (nk <= 64) return launch_ko1<D, 64>(q, kt, y, hs, out, pb, status, stream, launches);
  return launch_ko<D, 64>(q, kt, y, hs, out, pb, status, stream, launches);
}

// qt_per_item: the queries are the per-sub-item rows of a later step (else
// step one's Qt0); write_y: this is the last step (Y is written too).
template <int D, int NQ, bool PAIR>
cudaError_t launch_kr2(const bf16* qt0, const bf16* k, const bf16* v, bf16* kt, bf16* y,
                       float* hs, const Problem& pb, int* status, cudaStream_t stream,
                       int* launches, bool qt_per_item = false, bool write_y = false) {
  using L = KR2Layout<D, NQ, PAIR>;
  static std::once_flag attr_once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(attr_once, [] {
    attr_err = cudaFuncSetAttribute(kr2_kernel<D, NQ, PAIR>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes);
  });
  if (attr_err != cudaSuccess) return attr_err;
  CUtensorMap tq, tk, tv, tkt, tyy;
  {
    // paired tiles load each sub-item's b2 (<= 64) query rows as a 64-row box
    const cuuint64_t rows = (cuuint64_t)pb.G * pb.c1 * pb.b2 * (qt_per_item ? pb.b1 * pb.c2 : 1);
    const cuuint64_t dims[2] = {(cuuint64_t)D, rows};
    const cuuint64_t str[1] = {(cuuint64_t)D * 2};
    const cuuint32_t box[2] = {64, PAIR ? 64u : (cuuint32_t)kRows};
    if (!make_map(&tq, qt0, 2, dims, str, box)) return cudaErrorInvalidValue;
  }
  {
    if (!make_kv_map(&tk, k, pb, D, NQ) || !make_kv_map(&tv, v, pb, D, NQ))
      return cudaErrorInvalidValue;
  }
  const cuuint64_t ny = (cuuint64_t)pb.c1 * pb.b1 * pb.c2;
  {
    // Kt / Y [G][b2 i][c1 p][b1 k][c2 q][d] viewed as (d, c1*b1*c2, b2, G);
    // one warp's box is {64 columns, 1, 32 positions, 1}, clipped at b2
    const cuuint64_t dims[4] = {(cuuint64_t)D, ny, (cuuint64_t)pb.b2, (cuuint64_t)pb.G};
    const cuuint64_t str[3] = {(cuuint64_t)D * 2, ny * D * 2, ny * pb.b2 * D * 2};
    const cuuint32_t box[4] = {64, 1, 32, 1};
    if (!make_map(&tkt, kt, 4, dims, str, box)) return cudaErrorInvalidValue;
    if (!make_map(&tyy, y, 4, dims, str, box)) return cudaErrorInvalidValue;
  }
  KR2Args a;
  a.kt = kt;
  a.y = y;
  a.hs = hs;
  a.b1 = pb.b1;
  a.b2 = pb.b2;
  a.c1 = pb.c1;
  a.c2 = pb.c2;
  const long items = (long)pb.G * pb.c1 * pb.b1;
  if (items * pb.c2 >= (1L << 31)) return cudaErrorInvalidValue;
  if ((long)pb.G * pb.c1 * pb.b2 * pb.b1 * pb.c2 >= (1L << 31)) return cudaErrorInvalidValue;
  a.n_items = (int)items;
  a.write_y = (qt_per_item ? write_y : pb.T == 1) ? 1 : 0;
  a.qt_per_item = qt_per_item ? 1 : 0;
  a.sc_log2 = kLog2e * pb.sc;
  a.status = status;
  a.tr = pb.tr;
  a.real_lo = pb.real_lo;
  a.real_hi = pb.real_hi;
  const long units = (items * pb.c2 + L::kHalves - 1) / L::kHalves;
  const int grid = (int)std::min<long>(units, num_sms());
  return timed_launch("tc_r_update", stream, launches, [&] {
    return launch_pdl(kr2_kernel<D, NQ, PAIR>, dim3(grid), dim3(320), L::kBytes, stream, tq, tk,
                      tv, tkt, tyy, a);
  });
}

// Column-group tile width: the largest group (ceil(b2 / c2) keys) rounded up
// to 16, the K step of one tcgen05.mma.
inline int kr_group_tile(const Problem& pb) {
  return ((pb.b2 + pb.c2 - 1) / pb.c2 + 15) / 16 * 16;
}

template <int D>
cudaError_t launch_krl(const bf16* qt0, const bf16* k, const bf16* v, bf16* kt, bf16* y,
                       float* hs, const Problem& pb, int* status, cudaStream_t stream,
                       int* launches,
                       bool qt_per_item = false, bool write_y = false) {
  using L = KRLLayout<D>;
  static std::once_flag attr_once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(attr_once, [] {
    attr_err = cudaFuncSetAttribute(krl_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    L::kBytes);
  });
  if (attr_err != cudaSuccess) return attr_err;
  CUtensorMap tq, tk, tv, tkt, tyy;
  {
    const cuuint64_t rows = (cuuint64_t)pb.G * pb.c1 * pb.b2 * (qt_per_item ? pb.b1 * pb.c2 : 1);
    const cuuint64_t dims[2] = {(cuuint64_t)D, rows};
    const cuuint64_t str[1] = {(cuuint64_t)D * 2};
    const cuuint32_t box[2] = {64, kRows};
    if (!make_map(&tq, qt0, 2, dims, str, box)) return cudaErrorInvalidValue;
  }
  {
    if (!make_kv_map(&tk, k, pb, D, 128) || !make_kv_map(&tv, v, pb, D, 128))
      return cudaErrorInvalidValue;
  }
  {
    // Kt / Y viewed as (d, c1*b1*c2, b2, G); one warp's box {64, 1, 32, 1}, clipped at b2
    const cuuint64_t ny = (cuuint64_t)pb.c1 * pb.b1 * pb.c2;
    const cuuint64_t dims[4] = {(cuuint64_t)D, ny, (cuuint64_t)pb.b2, (cuuint64_t)pb.G};
    const cuuint64_t str[3] = {(cuuint64_t)D * 2, ny * D * 2, ny * pb.b2 * D * 2};
    const cuuint32_t box[4] = {64, 1, 32, 1};
    if (!make_map(&tkt, kt, 4, dims, str, box)) return cudaErrorInvalidValue;
    if (!make_map(&tyy, y, 4, dims, str, box)) return cudaErrorInvalidValue;
  }
  KRArgs a;
  a.kt = kt;
  a.y = y;
  a.hs = hs;
  a.b1 = pb.b1;
  a.b2 = pb.b2;
  a.c1 = pb.c1;
  a.c2 = pb.c2;
  a.write_y = (qt_per_item ? write_y : pb.T == 1) ? 1 : 0;
  a.qt_per_item = qt_per_item ? 1 : 0;
  a.sc_log2 = kLog2e * pb.sc;
  a.status = status;
  a.tr = pb.tr;
  a.real_lo = pb.real_lo;
  a.real_hi = pb.real_hi;
  a.n_itiles = (pb.b2 + kRows - 1) / kRows;
  const long items = (long)pb.G * pb.b1 * pb.c1 * a.n_itiles * pb.c2;
  if (items >= (1L << 31)) return cudaErrorInvalidValue;
  const int grid = (int)std::min<long>(items, num_sms());  // persistent: one CTA per SM
  return timed_launch("tc_r_update", stream, launches, [&] {
    return launch_pdl(krl_kernel<D>, dim3(grid), dim3(320), L::kBytes, stream, tq, tk, tv, tkt,
                      tyy, a, (int)items);
  });
}

template <int D>
cudaError_t launch_kl(const bf16* q, const bf16* kt, const float* hs, bf16* qt, const Problem& pb,
                      int* status, cudaStream_t stream, int* launches) {
  using L = KLLayout<D>;
  static std::once_flag attr_once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(attr_once, [] {
    attr_err =
        cudaFuncSetAttribute(kl_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes);
  });
  if (attr_err != cudaSuccess) return attr_err;
  const int nk = pb.b1 * pb.c2;
  const long key_rows = (long)pb.G * pb.b2 * pb.c1 * nk;
  CUtensorMap tq, tk;
  {
    if (!make_q_slab_map(&tq, q, pb, D)) return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)key_rows};
    const cuuint64_t str[1] = {(cuuint64_t)D * 2};
    const cuuint32_t box[2] = {64, 128};
    if (!make_map(&tk, kt, 2, dims, str, box)) return cudaErrorInvalidValue;
  }
  KLArgs a;
  a.hs = hs;
  a.qt = qt;
  a.b1 = pb.b1;
  a.b2 = pb.b2;
  a.c1 = pb.c1;
  a.c2 = pb.c2;
  a.nk = nk;
  a.real_lo = pb.real_lo;
  a.real_hi = pb.real_hi;
  a.sc = pb.sc;
  a.status = status;
  a.tr = pb.tr;
  const long blocks = (long)pb.G * pb.b2 * pb.c1;
  return timed_launch("tc_l_update", stream, launches, [&] {
    return launch_pdl(kl_kernel<D>, dim3((unsigned)blocks), dim3(256), L::kBytes, stream, tq, tk,
                      a);
  });
}

// Two-pass non-final L-update (rows of more than 128 keys or row groups of
// more than 128 rows): row log-sum-exps, then the aggregation per key tile.
template <int D>
cudaError_t launch_kl_two_pass(const bf16* q, const bf16* kt, const float* hs, float* lse,
                               bf16* qt, const Problem& pb, int* status, cudaStream_t stream,
                               int* launches) {
  using LS = KLSLayout<D>;
  using LM = KLMLayout<D>;
  static std::once_flag attr_once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(attr_once, [] {
    attr_err = cudaFuncSetAttribute(kls_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    LS::kBytes);
    if (attr_err == cudaSuccess)
      attr_err = cudaFuncSetAttribute(klm_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      LM::kBytes);
  });
  if (attr_err != cudaSuccess) return attr_err;
  const int nk = pb.b1 * pb.c2;
  const long key_rows = (long)pb.G * pb.b2 * pb.c1 * nk;
  CUtensorMap tq, tk;
  {
    if (!make_q_slab_map(&tq, q, pb, D)) return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)key_rows};
    const cuuint64_t str[1] = {(cuuint64_t)D * 2};
    const cuuint32_t box[2] = {64, 128};
    if (!make_map(&tk, kt, 2, dims, str, box)) return cudaErrorInvalidValue;
  }
  const int gmax = (pb.b1 + pb.c1 - 1) / pb.c1;
  KLSArgs as;
  as.hs = hs;
  as.lse = lse;
  as.b1 = pb.b1;
  as.b2 = pb.b2;
  as.c1 = pb.c1;
  as.nk = nk;
  as.row_tiles = (gmax + kRows - 1) / kRows;
  as.real_lo = pb.real_lo;
  as.real_hi = pb.real_hi;
  as.sc = pb.sc;
  as.status = status;
  as.tr = pb.tr;
  const long units = (long)pb.G * pb.b2 * pb.c1;
  if (units * as.row_tiles >= (1L << 31) || units * ((nk + 127) / 128) >= (1L << 31))
    return cudaErrorInvalidValue;
  cudaError_t e = timed_launch("tc_l_stats", stream, launches, [&] {
    return launch_pdl(kls_kernel<D>, dim3((unsigned)(units * as.row_tiles)), dim3(160),
                      LS::kBytes, stream, tq, tk, as);
  });
  if (e != cudaSuccess) return e;
  KLMArgs am;
  am.hs = hs;
  am.lse = lse;
  am.qt = qt;
  am.b1 = pb.b1;
  am.b2 = pb.b2;
  am.c1 = pb.c1;
  am.c2 = pb.c2;
  am.nk = nk;
  am.key_tiles = (nk + 127) / 128;
  am.real_lo = pb.real_lo;
  am.real_hi = pb.real_hi;
  am.sc = pb.sc;
  am.status = status;
  am.tr = pb.tr;
  return timed_launch("tc_l_update", stream, launches, [&] {
    return launch_pdl(klm_kernel<D>, dim3((unsigned)(units * am.key_tiles)), dim3(256),
                      LM::kBytes, stream, tq, tk, am);
  });
}

bool kl_single_tile(const Problem& pb) {
  return pb.b1 * pb.c2 <= 128 && (pb.b1 + pb.c1 - 1) / pb.c1 <= kRows;
}

// One later step: the non-final L-update (aggregated queries Qt of every
// sub-item), then the R-update from them.  The L-update takes one tile each
// way (rows of <= 128 keys, row groups of <= 128 rows) in one kernel, any
// other shape in the two-pass pair; the R-update takes the kernel step one
// takes for the same groups, reading each sub-item's own query rows.
template <int D>
cudaError_t launch_later_step(const bf16* q, const bf16* k, const bf16* v, bf16* qt, bf16* kt,
                              bf16* y, float* hs, float* lse, const Problem& pb, bool last,
                              int* status, cudaStream_t stream, int* launches) {
  cudaError_t e = kl_single_tile(pb)
                      ? launch_kl<D>(q, kt, hs, qt, pb, status, stream, launches)
                      : launch_kl_two_pass<D>(q, kt, hs, lse, qt, pb, status, stream, launches);
  if (e != cudaSuccess) return e;
  if (small_r_fits(pb)) return launch_small_r(qt, k, v, kt, y, hs, pb, true, last, stream, launches);
  if (kr_group_tile(pb) <= 96 && pb.b2 <= kRows) {
    switch (kr_group_tile(pb)) {
#define MONARCH_KR2_STEP(NQ)                                                                   \
  case NQ:                                                                                     \
    return pb.b2 <= 64 ? launch_kr2<D, NQ, true>(qt, k, v, kt, y, hs, pb, status, stream,     \
                                                 launches, true, last)                         \
                       : launch_kr2<D, NQ, false>(qt, k, v, kt, y, hs, pb, status, stream,    \
                                                  launches, true, last);
      MONARCH_KR2_STEP(16)
      MONARCH_KR2_STEP(32)
      MONARCH_KR2_STEP(48)
      MONARCH_KR2_STEP(64)
#define MONARCH_KR2_WIDE(NQ)                                                                    \
  case NQ:                                                                                      \
    return launch_kr2<D, NQ, false>(qt, k, v, kt, y, hs, pb, status, stream, launches, true, last);
      MONARCH_KR2_WIDE(80)
      MONARCH_KR2_WIDE(96)
#undef MONARCH_KR2_WIDE
#undef MONARCH_KR2_STEP
      default: return cudaErrorInvalidValue;
    }
  }
  return launch_krl<D>(qt, k, v, kt, y, hs, pb, status, stream, launches, true, last);
}

// Step one: aggregated queries under the uniform L, then the R-update: one
// warp per group on the CUDA cores for groups of <= 8 keys over <= 32
// positions, the paired-tile kernel for column groups of <= 96 keys over
// <= 128 positions (two groups per tile when b2 <= 64 and the groups hold
// <= 64 keys), the streaming kernel for wider groups or more positions.
template <int D>
cudaError_t launch_r_step1(const bf16* q, const bf16* k, const bf16* v, bf16* qt0, bf16* kt,
                           bf16* y, float* hs, const Problem& pb, int* status,
                           cudaStream_t stream, int* launches) {
  cudaError_t e =
      small_init_fits(pb)
          ? launch_small_init(q, qt0, pb, stream, launches)
          : timed_launch("tc_init_qt", stream, launches, [&] {
              // fewer units than SMs (a few long row groups): 32 warps per unit.
              // The thread count follows the whole call's units (see Problem).
              const long units = (long)pb.G * pb.c1 * pb.b2;
              const long shape_units = pb.init_units > 0 ? pb.init_units : units;
              if (shape_units < num_sms())
                return launch_pdl(init_qt_bf16_kernel<D, 1024>, dim3((unsigned)units),
                                  dim3(1024), 0, stream, q, qt0, pb);
              return shape_units <= 5L * num_sms()
                         ? launch_pdl(init_qt_bf16_kernel<D, 256>, dim3((unsigned)units),
                                      dim3(256), 0, stream, q, qt0, pb)
                         : launch_pdl(init_qt_bf16_kernel<D, 128>, dim3((unsigned)units),
                                      dim3(128), 0, stream, q, qt0, pb);
            });
  if (e != cudaSuccess) return e;
  // column groups of <= 8 keys over <= 32 positions: one warp per group
  if (small_r_fits(pb))
    return launch_small_r(qt0, k, v, kt, y, hs, pb, false, pb.T == 1, stream, launches);
  // column groups of <= 64 keys over <= 128 positions: the persistent kernel
  if (kr_group_tile(pb) <= 96 && pb.b2 <= kRows) {
    switch (kr_group_tile(pb)) {
#define MONARCH_KR2_CASE(NQ)                                                               \
  case NQ:                                                                                 \
    return pb.b2 <= 64                                                                     \
               ? launch_kr2<D, NQ, true>(qt0, k, v, kt, y, hs, pb, status, stream, launches) \
               : launch_kr2<D, NQ, false>(qt0, k, v, kt, y, hs, pb, status, stream, launches);
      MONARCH_KR2_CASE(16)
      MONARCH_KR2_CASE(32)
      MONARCH_KR2_CASE(48)
      MONARCH_KR2_CASE(64)
#define MONARCH_KR2_WIDE(NQ) \
  case NQ: return launch_kr2<D, NQ, false>(qt0, k, v, kt, y, hs, pb, status, stream, launches);
      MONARCH_KR2_WIDE(80)
      MONARCH_KR2_WIDE(96)
#undef MONARCH_KR2_WIDE
#undef MONARCH_KR2_CASE
      default: return cudaErrorInvalidValue;
    }
  }
  // wider groups, or more than 128 positions: the streaming kernel
  return launch_krl<D>(qt0, k, v, kt, y, hs, pb, status, stream, launches);
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

cudaError_t tc_selftest_timeout(int* status, unsigned long long limit_ns, cudaStream_t stream) {
  selftest_timeout_kernel<<<1, 32, 0, stream>>>(status, limit_ns);
  return cudaGetLastError();
}

bool tc_supports(const Problem& pb) {
  if (pb.d != 64 && pb.d != 128) return false;
  if (pb.T < 1) return false;
  const long key_rows = (long)pb.G * pb.b2 * pb.c1 * pb.b1 * pb.c2;
  if (key_rows + 256 >= (1L << 31) || (long)pb.G * pb.b1 >= (1L << 31)) return false;
  return encode_fn() != nullptr;
}

bool tc_takes_transposed(const Problem& pb) { return tc_supports(pb); }

bool tc_make_map(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims,
                 const cuuint64_t* strides, const cuuint32_t* box) {
  return make_map(m, base, rank, dims, strides, box);
}

bool tc_make_q_slab_map(CUtensorMap* m, const bf16* q, const Problem& pb, int D) {
  return make_q_slab_map(m, q, pb, D);
}

cudaError_t tc_step_one(const bf16* q, const bf16* k, const bf16* v, bf16* qt0, bf16* kt, bf16* y,
                        float* hs, const Problem& pb, int* status, cudaStream_t stream,
                        int* launches) {
  if (!tc_supports(pb)) return cudaErrorInvalidValue;
  return pb.d == 128
             ? launch_r_step1<128>(q, k, v, qt0, kt, y, hs, pb, status, stream, launches)
             : launch_r_step1<64>(q, k, v, qt0, kt, y, hs, pb, status, stream, launches);
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
  bf16* qt = reinterpret_cast<bf16*>(ws.qt);  // bf16 rows in the fp32-sized piece
  for (int t = 2; t <= pb.T; ++t) {
    e = pb.d == 128 ? launch_later_step<128>(q, k, v, qt, kt, y, ws.hs, ws.lse, pb, t == pb.T,
                                             status, stream, launches)
                    : launch_later_step<64>(q, k, v, qt, kt, y, ws.hs, ws.lse, pb, t == pb.T,
                                            status, stream, launches);
    if (e != cudaSuccess) return e;
  }
  if (pb.d == 128) return dispatch_ko<128>(q, kt, y, ws.hs, out, pb, status, stream, launches);
  return dispatch_ko<64>(q, kt, y, ws.hs, out, pb, status, stream, launches);
}

}  // namespace monarch
