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
// Kt, Y, Qt, P and L are stored as bf16 (as on the tensor-core path),
// softmax statistics and Hs in fp32.  Fragments come from shared memory by
// ldmatrix (transposed where the operand is stored k-major); bf16 rows are
// padded to 144 bytes (L tiles to 48) so that the 8 rows of each 8 x 8
// matrix hit different banks.
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

constexpr int kPL = 24;         // L tile row pitch (bf16): 48-byte rows, conflict-free ldmatrix

constexpr size_t smem_bytes(int n) {
  // Qs, Ks, Vs, Kt, Ys, Qt (bf16 rows), Hs, L tiles [16 positions][16 l][kPL] bf16
  return (size_t)n * 6 * kPB * 2 + (size_t)((n + 3) & ~3) * 4 + (size_t)kMaxB * kMaxB * kPL * 2;
}

// Four 8 x 8 bf16 matrices from shared memory (lane l gives the address of
// row l % 8 of matrix l / 8); .trans delivers each matrix transposed.
__device__ __forceinline__ void ldsm4(uint32_t (&r)[4], const bf16* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(tc::smem_u32(p)));
}

__device__ __forceinline__ void ldsm4_t(uint32_t (&r)[4], const bf16* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(tc::smem_u32(p)));
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
// (this thread: rows g and g+8, columns nt*8 + 2t + {0, 1}); columns outside
// [c_lo, c_hi) are masked, and so are columns already -inf.  On return s
// holds the normalised weights (all 0 in a row with every column masked);
// ent gets, per row half h, the entropy ln z - sum_j w_j (s_j - m) / z
// (-inf for such a row).
// MASKED (padded problems) also handles rows whose every column is masked.
template <bool MASKED>
__device__ __forceinline__ void quad_softmax(float (&s)[2][4], int c_lo, int c_hi, int t,
                                             float (&ent)[2]) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    float m = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int col = nt * 8 + 2 * t + e;
        if (col < c_lo || col >= c_hi) s[nt][2 * h + e] = -INFINITY;
        m = fmaxf(m, s[nt][2 * h + e]);
      }
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
    if (MASKED && m == -INFINITY) m = 0.f;  // every column masked: all weights 0
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
    const float inv = (!MASKED || z > 0.f) ? 1.f / z : 0.f;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) s[nt][2 * h + e] *= inv;
    ent[h] = (!MASKED || z > 0.f) ? __logf(z) - dot * inv : -INFINITY;
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

// Padding: the head's real tokens are grid tokens [real_lo, real_hi); q, k, v
// and out hold only those rows (real_hi - real_lo per head), pad rows are
// zero in shared memory and are masked in every softmax and aggregation.
// PADDED selects the masked instantiation; unpadded heads (real_lo = 0,
// real_hi = N) run the one without masks.
template <bool PADDED>
__global__ void __launch_bounds__(kThreads, 1)
    small_head_kernel(const bf16* __restrict__ q, const bf16* __restrict__ k,
                      const bf16* __restrict__ v, bf16* __restrict__ out, int b1, int b2, int T,
                      float sc, int real_lo, int real_hi) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int N = b1 * b2;
  auto real_tok = [&](int m) { return !PADDED || (m >= real_lo && m < real_hi); };
  const int n_src = real_hi - real_lo;  // rows per head in q, k, v, out
  bf16* Qs = reinterpret_cast<bf16*>(smem);  // token rows l * b2 + i
  bf16* Ks = Qs + N * kPB;
  bf16* Vs = Ks + N * kPB;
  bf16* Kt = Vs + N * kPB;                   // rows (i, k): i * b1 + k
  bf16* Ys = Kt + N * kPB;
  bf16* Qt = Ys + N * kPB;                   // rows (k, i): k * b2 + i
  float* Hs = reinterpret_cast<float*>(Qt + N * kPB);  // (i, k)
  bf16* Ls = reinterpret_cast<bf16*>(Hs + ((N + 3) & ~3));  // [position i][l][k], pitch kPL
  const long gh = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  // ldmatrix lane roles: matrix mi = lane / 8, row lr = lane % 8
  const int mi = lane >> 3, lr = lane & 7;

  // q, k, v of the head into shared memory (16-byte chunks); pad rows are zero
  {
    const uint4* gq = reinterpret_cast<const uint4*>(q + gh * n_src * kD);
    const uint4* gk = reinterpret_cast<const uint4*>(k + gh * n_src * kD);
    const uint4* gv = reinterpret_cast<const uint4*>(v + gh * n_src * kD);
    for (int x = tid; x < N * (kD / 8); x += kThreads) {
      const int r = x / (kD / 8), c = x % (kD / 8);
      const int so = r * kPB + c * 8;
      const bool real = real_tok(r);
      const int xs = (r - real_lo) * (kD / 8) + c;
      const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
      *reinterpret_cast<uint4*>(Qs + so) = real ? __ldg(gq + xs) : zero;
      *reinterpret_cast<uint4*>(Ks + so) = real ? __ldg(gk + xs) : zero;
      *reinterpret_cast<uint4*>(Vs + so) = real ? __ldg(gv + xs) : zero;
    }
  }
  __syncthreads();
  // step-one aggregated queries (uniform L): every row (k, i) gets the mean of
  // the real q_(l,i) (0 if position i has none)
  for (int x = tid; x < b2 * (kD / 2); x += kThreads) {
    const int i = x / (kD / 2), c = (x % (kD / 2)) * 2;
    float s0 = 0.f, s1 = 0.f;
    int nl = 0;
    for (int l = 0; l < b1; ++l) {
      if (!real_tok(l * b2 + i)) continue;
      const __nv_bfloat162 p = *reinterpret_cast<const __nv_bfloat162*>(Qs + (l * b2 + i) * kPB + c);
      s0 += __low2float(p);
      s1 += __high2float(p);
      ++nl;
    }
    const float inv_n = nl > 0 ? 1.f / (float)nl : 0.f;
    const uint32_t m = (!PADDED || nl == b1) ? tc::pack_bf16x2(s0 / (float)b1, s1 / (float)b1)
                                : tc::pack_bf16x2(s0 * inv_n, s1 * inv_n);
    for (int kk = 0; kk < b1; ++kk) *reinterpret_cast<uint32_t*>(Qt + (kk * b2 + i) * kPB + c) = m;
  }
  __syncthreads();

  for (int step = 1; step <= T; ++step) {
    const bool last = step == T;
    // ---- R-update: warp kk, rows i (positions), columns j (keys of chunk kk) ----
    if (warp < b1) {
      const int kk = warp;
      const bf16* kr = Ks + kk * b2 * kPB;
      const bf16* vr = Vs + kk * b2 * kPB;
      // A rows i (clamped; their results are unused), B rows j (keys, clamped and masked)
      const bf16* a_src = Qt + (kk * b2 + min(lr + (mi & 1) * 8, b2 - 1)) * kPB + (mi >> 1) * 8;
      const bf16* b_src = kr + min(lr + (mi >> 1) * 8, b2 - 1) * kPB + (mi & 1) * 8;
      float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
      for (int ks = 0; ks < kD / 16; ++ks) {
        uint32_t a[4], b[4];
        ldsm4(a, a_src + ks * 16);
        ldsm4(b, b_src + ks * 16);
        mma16816(s[0], a, b[0], b[1]);
        mma16816(s[1], a, b[2], b[3]);
      }
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) s[nt][e] *= sc;
      // real keys of chunk kk: j in [j_lo, j_hi)
      const int j_lo = min(max(real_lo - kk * b2, 0), b2);
      const int j_hi = max(min(real_hi - kk * b2, b2), j_lo);
      float ent[2];
      quad_softmax<PADDED>(s, j_lo, j_hi, t, ent);
      if (t == 0) {
        if (g < b2) Hs[g * b1 + kk] = ent[0];
        if (g + 8 < b2) Hs[(g + 8) * b1 + kk] = ent[1];
      }
      uint32_t pa[4];
      acc_to_a(s, pa);  // R (rows i, k-dim j)
      // B[j][c] = k_(kk,j)[c] (stored j-major): transposed ldmatrix, two 8-column tiles per load
      const int jb = min(lr + (mi & 1) * 8, b2 - 1);
#pragma unroll
      for (int cb = 0; cb < kD / 16; ++cb) {
        const int coff = cb * 16 + (mi >> 1) * 8;
        uint32_t b[4];
        ldsm4_t(b, kr + jb * kPB + coff);
        float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        mma16816(acc[0], pa, b[0], b[1]);
        mma16816(acc[1], pa, b[2], b[3]);
        float ay[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        if (last) {
          ldsm4_t(b, vr + jb * kPB + coff);
          mma16816(ay[0], pa, b[0], b[1]);
          mma16816(ay[1], pa, b[2], b[3]);
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int cc = cb * 16 + h * 8 + 2 * t;
          if (g < b2) {
            *reinterpret_cast<uint32_t*>(Kt + (g * b1 + kk) * kPB + cc) =
                tc::pack_bf16x2(acc[h][0], acc[h][1]);
            if (last)
              *reinterpret_cast<uint32_t*>(Ys + (g * b1 + kk) * kPB + cc) =
                  tc::pack_bf16x2(ay[h][0], ay[h][1]);
          }
          if (g + 8 < b2) {
            *reinterpret_cast<uint32_t*>(Kt + ((g + 8) * b1 + kk) * kPB + cc) =
                tc::pack_bf16x2(acc[h][2], acc[h][3]);
            if (last)
              *reinterpret_cast<uint32_t*>(Ys + ((g + 8) * b1 + kk) * kPB + cc) =
                  tc::pack_bf16x2(ay[h][2], ay[h][3]);
          }
        }
      }
    }
    __syncthreads();
    // ---- L-update: warp i, rows l, columns k ----
    if (warp < b2) {
      const int i = warp;
      const bf16* ktr = Kt + i * b1 * kPB;
      // A rows l (query rows of position i, clamped), B rows k (Kt rows, clamped and masked)
      const bf16* a_src = Qs + (min(lr + (mi & 1) * 8, b1 - 1) * b2 + i) * kPB + (mi >> 1) * 8;
      const bf16* b_src = ktr + min(lr + (mi >> 1) * 8, b1 - 1) * kPB + (mi & 1) * 8;
      float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
      for (int ks = 0; ks < kD / 16; ++ks) {
        uint32_t a[4], b[4];
        ldsm4(a, a_src + ks * 16);
        ldsm4(b, b_src + ks * 16);
        mma16816(s[0], a, b[0], b[1]);
        mma16816(s[1], a, b[2], b[3]);
      }
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int col = min(nt * 8 + 2 * t + (e & 1), b1 - 1);
          s[nt][e] = fmaf(s[nt][e], sc, Hs[i * b1 + col]);
        }
      float ent[2];
      quad_softmax<PADDED>(s, 0, b1, t, ent);  // chunks without a real key carry Hs = -inf
      if (!last) {
        // L (bf16; rows l >= b1 zeroed) to this position's tile, then
        // Qt = L^T q / column sums of L
        bf16* Lt = Ls + i * kMaxB * kPL;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int row = g + 8 * h, col = nt * 8 + 2 * t;
            const bool real = row < b1 && real_tok(row * b2 + i);
            *reinterpret_cast<uint32_t*>(Lt + row * kPL + col) =
                real ? tc::pack_bf16x2(s[nt][2 * h], s[nt][2 * h + 1]) : 0u;
          }
        __syncwarp();
        // A = L^T (rows k, k-dim l) from the l-major tile: transposed ldmatrix
        uint32_t a[4];
        ldsm4_t(a, Lt + (lr + (mi >> 1) * 8) * kPL + (mi & 1) * 8);
        float cs0 = 0.f, cs1 = 0.f;  // column sums for k = g, g + 8 (of the bf16 weights)
        for (int l = 0; l < b1; ++l) {
          cs0 += __bfloat162float(Lt[l * kPL + g]);
          cs1 += __bfloat162float(Lt[l * kPL + g + 8]);
        }
        const float inv0 = cs0 > 0.f ? 1.f / cs0 : 0.f, inv1 = cs1 > 0.f ? 1.f / cs1 : 0.f;
        // B[l][c] = q_(l,i)[c] (stored l-major): transposed ldmatrix; rows l >= b1 clamped
        // (their A weights are 0)
        const bf16* qb_src = Qs + (min(lr + (mi & 1) * 8, b1 - 1) * b2 + i) * kPB + (mi >> 1) * 8;
#pragma unroll
        for (int cb = 0; cb < kD / 16; ++cb) {
          uint32_t b[4];
          ldsm4_t(b, qb_src + cb * 16);
          float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
          mma16816(acc[0], a, b[0], b[1]);
          mma16816(acc[1], a, b[2], b[3]);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int cc = cb * 16 + h * 8 + 2 * t;
            if (g < b1)
              *reinterpret_cast<uint32_t*>(Qt + (g * b2 + i) * kPB + cc) =
                  tc::pack_bf16x2(acc[h][0] * inv0, acc[h][1] * inv0);
            if (g + 8 < b1)
              *reinterpret_cast<uint32_t*>(Qt + ((g + 8) * b2 + i) * kPB + cc) =
                  tc::pack_bf16x2(acc[h][2] * inv1, acc[h][3] * inv1);
          }
        }
      } else {
        // O_(l,i) = L Y_i: A = L (rows l, k-dim k), B[k][c] = Y_{i,k}[c] (stored
        // k-major): transposed ldmatrix; rows k >= b1 clamped (their L weights are 0)
        uint32_t a[4];
        acc_to_a(s, a);
        const bf16* y_src = Ys + (i * b1 + min(lr + (mi & 1) * 8, b1 - 1)) * kPB + (mi >> 1) * 8;
        // only real rows are written, to their row in the unpadded output
        const int m0 = g * b2 + i, m1 = (g + 8) * b2 + i;
        const bool w0 = g < b1 && real_tok(m0);
        const bool w1 = g + 8 < b1 && real_tok(m1);
        bf16* orow0 = out + (gh * n_src + (m0 - real_lo)) * kD;
        bf16* orow1 = out + (gh * n_src + (m1 - real_lo)) * kD;
#pragma unroll
        for (int cb = 0; cb < kD / 16; ++cb) {
          uint32_t b[4];
          ldsm4_t(b, y_src + cb * 16);
          float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
          mma16816(acc[0], a, b[0], b[1]);
          mma16816(acc[1], a, b[2], b[3]);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int cc = cb * 16 + h * 8 + 2 * t;
            if (w0) *reinterpret_cast<uint32_t*>(orow0 + cc) = tc::pack_bf16x2(acc[h][0], acc[h][1]);
            if (w1) *reinterpret_cast<uint32_t*>(orow1 + cc) = tc::pack_bf16x2(acc[h][2], acc[h][3]);
          }
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
    attr = cudaFuncSetAttribute(small_head_kernel<false>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_bytes(kMaxN));
    if (attr == cudaSuccess)
      attr = cudaFuncSetAttribute(small_head_kernel<true>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)smem_bytes(kMaxN));
  });
  if (attr != cudaSuccess) return attr;
  if (!small_head_supports(pb)) return cudaErrorInvalidValue;
  const size_t smem = smem_bytes(pb.b1 * pb.b2);
  return timed_launch("small_head", stream, launches, [&] {
    if (is_padded(pb))
      small_head_kernel<true><<<pb.G, kThreads, smem, stream>>>(q, k, v, out, pb.b1, pb.b2, pb.T,
                                                                pb.sc, pb.real_lo, pb.real_hi);
    else
      small_head_kernel<false><<<pb.G, kThreads, smem, stream>>>(q, k, v, out, pb.b1, pb.b2, pb.T,
                                                                 pb.sc, pb.real_lo, pb.real_hi);
  });
}

}  // namespace monarch
