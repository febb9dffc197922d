// One CTA per head for small untiled heads (b1, b2 <= 16, d = 64, any T):
// q, k, v and every intermediate (aggregated queries Qt, Kt, Y, entropies
// Hs, L weights) stay in shared memory for all T alternating steps, so the
// only global traffic is q, k, v in and O out (MonarchAttention OpenReview
// discussion, the alternating maximisation; uniform initial L).  Every block
// product is at most 16 x 16 x 64, far below a tcgen05 tile, so each warp
// runs it on the tensor cores with warp-level mma.sync (m16n8k16, bf16 in,
// fp32 accumulate), FlashAttention-2 style: the softmax works on the
// accumulator fragments and P goes back in as the A fragment.
//   init      Qt_{k,i} = mean_l q_(l,i) for every k
//   R-update  warp k:  S = sc Qt_k K_k^T (rows i, columns j), R = softmax_j,
//             Hs = entropy of each R row, Kt_{i,k} = R K_k, Y_{i,k} = R V_k
//             (last step)
//   L-update  warp i:  S = sc q_(.,i) Kt_i^T + Hs_i (rows l, columns k),
//             L = softmax_k; non-final: Qt_{k,i} = L^T q_(.,i) / column sums
//             of L; final: O_(l,i) = L Y_i
// Kt, Y, Qt and P are stored as bf16 (as on the tensor-core path), softmax
// statistics and Hs in fp32.  bf16 rows are padded to 144 bytes so that the
// 8 row groups of a fragment load hit different shared-memory banks.
#include "small_head.cuh"

#include <mutex>

#include "tc_ptx.cuh"
#include "timing.cuh"

namespace monarch {
namespace {

constexpr int kD = 64;
constexpr int kMaxB = 16;
constexpr int kMaxN = 216;
constexpr int kPB = 72;        // bf16 row pitch (elements)
constexpr int kWarps = 16;     // one per chunk k (R-update) or position i (L-update)
constexpr int kThreads = kWarps * 32;
constexpr float kLog2e = 1.4426950408889634f;

constexpr size_t smem_bytes(int n) {
  // Qs, Ks, Vs, Kt, Ys, Qt (bf16 rows), Hs, L tiles [16 positions][16][16] fp32
  return (size_t)n * (6 * kPB * 2 + 4) + (size_t)kMaxB * kMaxB * kMaxB * 4;
}

__device__ __forceinline__ uint32_t ld32(const bf16* p) {
  return *reinterpret_cast<const uint32_t*>(p);
}

__device__ __forceinline__ uint32_t pack2(bf16 lo, bf16 hi) {
  return (uint32_t)__bfloat16_as_ushort(lo) | ((uint32_t)__bfloat16_as_ushort(hi) << 16);
}

// D += A B for one m16n8k16 tile (A 16 x 16 row-major, B 16 x 8 column-major).
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Row softmax over the 16 columns of a 16 x 16 accumulator pair s[2][4]
// (this thread: rows g and g+8, columns nt*8 + 2t + {0, 1}); columns >= n
// are masked.  On return s holds the normalised weights; lnz/dot get, per
// row half h, ln z and sum_j w_j (s_j - m) (for the entropy).
__device__ __forceinline__ void quad_softmax(float (&s)[2][4], int n, int t, float (&ent)[2]) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    float m = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int col = nt * 8 + 2 * t + e;
        if (col >= n) s[nt][2 * h + e] = -INFINITY;
        m = fmaxf(m, s[nt][2 * h + e]);
      }
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
    float z = 0.f, dot = 0.f;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float x = s[nt][2 * h + e];
        const float w = tc::ex2((x - m) * kLog2e);  // 0 for masked columns
        if (w > 0.f) dot += w * (x - m);
        z += w;
        s[nt][2 * h + e] = w;
      }
    z += __shfl_xor_sync(0xffffffffu, z, 1);
    z += __shfl_xor_sync(0xffffffffu, z, 2);
    dot += __shfl_xor_sync(0xffffffffu, dot, 1);
    dot += __shfl_xor_sync(0xffffffffu, dot, 2);
    const float inv = 1.f / z;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) s[nt][2 * h + e] *= inv;
    ent[h] = __logf(z) - dot * inv;
  }
}

// The accumulator pair s[2][4] (16 x 16) as the bf16 A fragment of the next
// product (its columns become the K dimension).
__device__ __forceinline__ void acc_to_a(const float (&s)[2][4], uint32_t (&a)[4]) {
  a[0] = tc::pack_bf16x2(s[0][0], s[0][1]);
  a[1] = tc::pack_bf16x2(s[0][2], s[0][3]);
  a[2] = tc::pack_bf16x2(s[1][0], s[1][1]);
  a[3] = tc::pack_bf16x2(s[1][2], s[1][3]);
}

__global__ void __launch_bounds__(kThreads, 1)
    small_head_kernel(const bf16* __restrict__ q, const bf16* __restrict__ k,
                      const bf16* __restrict__ v, bf16* __restrict__ out, int b1, int b2, int T,
                      float sc) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int N = b1 * b2;
  bf16* Qs = reinterpret_cast<bf16*>(smem);  // token rows l * b2 + i
  bf16* Ks = Qs + N * kPB;
  bf16* Vs = Ks + N * kPB;
  bf16* Kt = Vs + N * kPB;                   // rows (i, k): i * b1 + k
  bf16* Ys = Kt + N * kPB;
  bf16* Qt = Ys + N * kPB;                   // rows (k, i): k * b2 + i
  float* Hs = reinterpret_cast<float*>(Qt + N * kPB);  // (i, k)
  float* Ls = Hs + N;                        // [position i][l][k] L tiles
  const long gh = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;

  // q, k, v of the head into shared memory (16-byte chunks)
  {
    const uint4* gq = reinterpret_cast<const uint4*>(q + gh * N * kD);
    const uint4* gk = reinterpret_cast<const uint4*>(k + gh * N * kD);
    const uint4* gv = reinterpret_cast<const uint4*>(v + gh * N * kD);
    for (int x = tid; x < N * (kD / 8); x += kThreads) {
      const int r = x / (kD / 8), c = x % (kD / 8);
      const int so = r * kPB + c * 8;
      *reinterpret_cast<uint4*>(Qs + so) = __ldg(gq + x);
      *reinterpret_cast<uint4*>(Ks + so) = __ldg(gk + x);
      *reinterpret_cast<uint4*>(Vs + so) = __ldg(gv + x);
    }
  }
  __syncthreads();
  // step-one aggregated queries (uniform L): every row (k, i) gets mean_l q_(l,i)
  for (int x = tid; x < b2 * (kD / 2); x += kThreads) {
    const int i = x / (kD / 2), c = (x % (kD / 2)) * 2;
    float s0 = 0.f, s1 = 0.f;
    for (int l = 0; l < b1; ++l) {
      const __nv_bfloat162 p = *reinterpret_cast<const __nv_bfloat162*>(Qs + (l * b2 + i) * kPB + c);
      s0 += __low2float(p);
      s1 += __high2float(p);
    }
    const uint32_t m = tc::pack_bf16x2(s0 / (float)b1, s1 / (float)b1);
    for (int kk = 0; kk < b1; ++kk) *reinterpret_cast<uint32_t*>(Qt + (kk * b2 + i) * kPB + c) = m;
  }
  __syncthreads();

  for (int step = 1; step <= T; ++step) {
    const bool last = step == T;
    // ---- R-update: warp kk, rows i (positions), columns j (keys of chunk kk) ----
    if (warp < b1) {
      const int kk = warp;
      const int i0 = min(g, b2 - 1), i1 = min(g + 8, b2 - 1);  // clamped rows (results unused)
      const bf16* qa = Qt + (kk * b2 + i0) * kPB;
      const bf16* qb = Qt + (kk * b2 + i1) * kPB;
      const bf16* kr = Ks + kk * b2 * kPB;
      const bf16* vr = Vs + kk * b2 * kPB;
      float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
      for (int ks = 0; ks < kD / 16; ++ks) {
        const int c = ks * 16 + 2 * t;
        const uint32_t a[4] = {ld32(qa + c), ld32(qb + c), ld32(qa + c + 8), ld32(qb + c + 8)};
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          const bf16* krow = kr + min(nt * 8 + g, b2 - 1) * kPB;
          mma16816(s[nt], a, ld32(krow + c), ld32(krow + c + 8));
        }
      }
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) s[nt][e] *= sc;
      float ent[2];
      quad_softmax(s, b2, t, ent);
      if (t == 0) {
        if (g < b2) Hs[g * b1 + kk] = ent[0];
        if (g + 8 < b2) Hs[(g + 8) * b1 + kk] = ent[1];
      }
      uint32_t pa[4];
      acc_to_a(s, pa);  // R (rows i, k-dim j)
      // B[j][c] = k_(kk,j)[c]: rows j = 2t, 2t+1 (+8), column c = nt*8 + g
      const int j0 = min(2 * t, b2 - 1), j1 = min(2 * t + 1, b2 - 1);
      const int j2 = min(2 * t + 8, b2 - 1), j3 = min(2 * t + 9, b2 - 1);
#pragma unroll
      for (int nt = 0; nt < kD / 8; ++nt) {
        const int c = nt * 8 + g;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        mma16816(acc, pa, pack2(kr[j0 * kPB + c], kr[j1 * kPB + c]),
                 pack2(kr[j2 * kPB + c], kr[j3 * kPB + c]));
        const int cc = nt * 8 + 2 * t;
        if (g < b2)
          *reinterpret_cast<uint32_t*>(Kt + (g * b1 + kk) * kPB + cc) = tc::pack_bf16x2(acc[0], acc[1]);
        if (g + 8 < b2)
          *reinterpret_cast<uint32_t*>(Kt + ((g + 8) * b1 + kk) * kPB + cc) =
              tc::pack_bf16x2(acc[2], acc[3]);
        if (last) {
          float ay[4] = {0.f, 0.f, 0.f, 0.f};
          mma16816(ay, pa, pack2(vr[j0 * kPB + c], vr[j1 * kPB + c]),
                   pack2(vr[j2 * kPB + c], vr[j3 * kPB + c]));
          if (g < b2)
            *reinterpret_cast<uint32_t*>(Ys + (g * b1 + kk) * kPB + cc) = tc::pack_bf16x2(ay[0], ay[1]);
          if (g + 8 < b2)
            *reinterpret_cast<uint32_t*>(Ys + ((g + 8) * b1 + kk) * kPB + cc) =
                tc::pack_bf16x2(ay[2], ay[3]);
        }
      }
    }
    __syncthreads();
    // ---- L-update: warp i, rows l, columns k ----
    if (warp < b2) {
      const int i = warp;
      const int l0 = min(g, b1 - 1), l1 = min(g + 8, b1 - 1);
      const bf16* qa = Qs + (l0 * b2 + i) * kPB;
      const bf16* qb = Qs + (l1 * b2 + i) * kPB;
      const bf16* ktr = Kt + i * b1 * kPB;
      float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
      for (int ks = 0; ks < kD / 16; ++ks) {
        const int c = ks * 16 + 2 * t;
        const uint32_t a[4] = {ld32(qa + c), ld32(qb + c), ld32(qa + c + 8), ld32(qb + c + 8)};
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          const bf16* krow = ktr + min(nt * 8 + g, b1 - 1) * kPB;
          mma16816(s[nt], a, ld32(krow + c), ld32(krow + c + 8));
        }
      }
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int col = min(nt * 8 + 2 * t + (e & 1), b1 - 1);
          s[nt][e] = fmaf(s[nt][e], sc, Hs[i * b1 + col]);
        }
      float ent[2];
      quad_softmax(s, b1, t, ent);
      if (!last) {
        // L (rows l >= b1 zeroed) to this position's tile, then Qt = L^T q / colsum(L)
        float* Lt = Ls + i * kMaxB * kMaxB;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int row = g + 8 * (e >> 1), col = nt * 8 + 2 * t + (e & 1);
            Lt[row * kMaxB + col] = row < b1 ? s[nt][e] : 0.f;
          }
        __syncwarp();
        // A = L^T: rows k = g, g+8; k-dim l = 2t, 2t+1 (+8)
        uint32_t a[4];
        {
          auto lk = [&](int l, int kk) { return __float2bfloat16_rn(Lt[l * kMaxB + kk]); };
          a[0] = pack2(lk(2 * t, g), lk(2 * t + 1, g));
          a[1] = pack2(lk(2 * t, g + 8), lk(2 * t + 1, g + 8));
          a[2] = pack2(lk(2 * t + 8, g), lk(2 * t + 9, g));
          a[3] = pack2(lk(2 * t + 8, g + 8), lk(2 * t + 9, g + 8));
        }
        float cs0 = 0.f, cs1 = 0.f;  // column sums for k = g, g + 8
        for (int l = 0; l < b1; ++l) {
          cs0 += Lt[l * kMaxB + g];
          cs1 += Lt[l * kMaxB + g + 8];
        }
        const float inv0 = cs0 > 0.f ? 1.f / cs0 : 0.f, inv1 = cs1 > 0.f ? 1.f / cs1 : 0.f;
        // B[l][c] = q_(l,i)[c]: rows l = 2t, 2t+1 (+8), column c = nt*8 + g
        const int r0 = min(2 * t, b1 - 1) * b2 + i, r1 = min(2 * t + 1, b1 - 1) * b2 + i;
        const int r2 = min(2 * t + 8, b1 - 1) * b2 + i, r3 = min(2 * t + 9, b1 - 1) * b2 + i;
#pragma unroll
        for (int nt = 0; nt < kD / 8; ++nt) {
          const int c = nt * 8 + g;
          float acc[4] = {0.f, 0.f, 0.f, 0.f};
          mma16816(acc, a, pack2(Qs[r0 * kPB + c], Qs[r1 * kPB + c]),
                   pack2(Qs[r2 * kPB + c], Qs[r3 * kPB + c]));
          const int cc = nt * 8 + 2 * t;
          if (g < b1)
            *reinterpret_cast<uint32_t*>(Qt + (g * b2 + i) * kPB + cc) =
                tc::pack_bf16x2(acc[0] * inv0, acc[1] * inv0);
          if (g + 8 < b1)
            *reinterpret_cast<uint32_t*>(Qt + ((g + 8) * b2 + i) * kPB + cc) =
                tc::pack_bf16x2(acc[2] * inv1, acc[3] * inv1);
        }
      } else {
        // O_(l,i) = L Y_i: A = L (rows l, k-dim k), B[k][c] = Y_{i,k}[c]
        uint32_t a[4];
        acc_to_a(s, a);
        const bf16* yr = Ys + i * b1 * kPB;
        const int k0 = min(2 * t, b1 - 1), k1 = min(2 * t + 1, b1 - 1);
        const int k2 = min(2 * t + 8, b1 - 1), k3 = min(2 * t + 9, b1 - 1);
        bf16* orow0 = out + (gh * N + g * b2 + i) * kD;
        bf16* orow1 = out + (gh * N + (g + 8) * b2 + i) * kD;
#pragma unroll
        for (int nt = 0; nt < kD / 8; ++nt) {
          const int c = nt * 8 + g;
          float acc[4] = {0.f, 0.f, 0.f, 0.f};
          mma16816(acc, a, pack2(yr[k0 * kPB + c], yr[k1 * kPB + c]),
                   pack2(yr[k2 * kPB + c], yr[k3 * kPB + c]));
          const int cc = nt * 8 + 2 * t;
          if (g < b1) *reinterpret_cast<uint32_t*>(orow0 + cc) = tc::pack_bf16x2(acc[0], acc[1]);
          if (g + 8 < b1) *reinterpret_cast<uint32_t*>(orow1 + cc) = tc::pack_bf16x2(acc[2], acc[3]);
        }
      }
    }
    __syncthreads();
  }
}

}  // namespace

bool small_head_supports(const Problem& pb) {
  return pb.d == kD && pb.c1 == 1 && pb.c2 == 1 && pb.T >= 1 && pb.b1 <= kMaxB &&
         pb.b2 <= kMaxB && pb.b1 * pb.b2 <= kMaxN;
}

cudaError_t small_head_forward(const bf16* q, const bf16* k, const bf16* v, bf16* out,
                               const Problem& pb, cudaStream_t stream, int* launches) {
  static std::once_flag once;
  static cudaError_t attr = cudaSuccess;
  std::call_once(once, [] {
    attr = cudaFuncSetAttribute(small_head_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)smem_bytes(kMaxN));
  });
  if (attr != cudaSuccess) return attr;
  if (!small_head_supports(pb)) return cudaErrorInvalidValue;
  const size_t smem = smem_bytes(pb.b1 * pb.b2);
  return timed_launch("small_head", stream, launches, [&] {
    small_head_kernel<<<pb.G, kThreads, smem, stream>>>(q, k, v, out, pb.b1, pb.b2, pb.T, pb.sc);
  });
}

}  // namespace monarch
