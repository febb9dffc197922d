// One CTA per head for small untiled heads (b1, b2 <= 16, d = 64, any T):
// q, k, v and every intermediate (aggregated queries Qt, Kt, Y, entropies
// Hs, L weights) stay in shared memory for all T alternating steps, so the
// only global traffic is q, k, v in and O out.  Four consecutive threads own
// one softmax row of each half-step (16 of the 64 columns each, dot products
// combined by warp shuffles) (MonarchAttention OpenReview discussion, the
// alternating maximisation; uniform initial L):
//   init      Qt_{k,i} = mean_l q_(l,i) for every k
//   R-update  row (k, i):  s_j = sc Qt_{k,i} . k_(k,j), R = softmax_j(s),
//             Hs = entropy of R, Kt_{i,k} = sum_j R_j k_(k,j),
//             Y_{i,k} = sum_j R_j v_(k,j) (last step)
//   L-update  row (i, l):  s_k = sc q_(l,i) . Kt_{i,k} + Hs_{i,k},
//             L = softmax_k(s); non-final: L to shared memory, then row
//             (k, i): Qt_{k,i} = sum_l L_{l,k} q_(l,i) / sum_l L_{l,k};
//             final: O_(l,i) = sum_k L_k Y_{i,k}
// Arithmetic is fp32; Kt and Y are stored as bf16 (as on the tensor-core
// path), Qt in fp32.  Rows are padded (144-byte bf16 rows, 272-byte fp32
// rows) so that threads reading different rows at one column hit different
// shared-memory banks.
#include "small_head.cuh"

#include <algorithm>
#include <mutex>

#include "tc_ptx.cuh"
#include "timing.cuh"

namespace monarch {
namespace {

constexpr int kD = 64;
constexpr int kMaxB = 16;
constexpr int kMaxN = 216;
constexpr int kPB = 72;   // bf16 row pitch (elements)
constexpr int kPF = 68;   // fp32 row pitch (elements)
constexpr int kParts = 4;                          // threads per row
constexpr int kChunks = kD / 8 / kParts;           // 8-column chunks per thread
constexpr int kThreads = (kMaxN * kParts + 31) / 32 * 32;
constexpr float kLog2e = 1.4426950408889634f;

constexpr size_t smem_bytes(int n) {
  return (size_t)n * (5 * kPB * 2 + kPF * 4 + 4 + kMaxB * 4);
}

__device__ __forceinline__ void unpack8(const uint4& u, float (&x)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    x[2 * e] = __uint_as_float(w[e] << 16);
    x[2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
  }
}

__device__ __forceinline__ uint4 pack8(const float (&x)[8]) {
  uint4 u;
  u.x = tc::pack_bf16x2(x[0], x[1]);
  u.y = tc::pack_bf16x2(x[2], x[3]);
  u.z = tc::pack_bf16x2(x[4], x[5]);
  u.w = tc::pack_bf16x2(x[6], x[7]);
  return u;
}

// softmax of s[0..n) in place (natural-log logits); returns ln(sum exp(s - max))
// and writes the max to *m
__device__ __forceinline__ float softmax16(float (&s)[kMaxB], int n, float* m) {
  float mx = -INFINITY;
#pragma unroll
  for (int j = 0; j < kMaxB; ++j)
    if (j < n) mx = fmaxf(mx, s[j]);
  float z = 0.f;
#pragma unroll
  for (int j = 0; j < kMaxB; ++j) {
    s[j] = j < n ? tc::ex2((s[j] - mx) * kLog2e) : 0.f;
    z += s[j];
  }
  *m = mx;
  return z;
}

__global__ void __launch_bounds__(kThreads, 1)
    small_head_kernel(const bf16* __restrict__ q, const bf16* __restrict__ k,
                      const bf16* __restrict__ v, bf16* __restrict__ out, int b1, int b2, int T,
                      float sc) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int N = b1 * b2;
  bf16* Qs = reinterpret_cast<bf16*>(smem);  // token rows
  bf16* Ks = Qs + N * kPB;
  bf16* Vs = Ks + N * kPB;
  bf16* Kt = Vs + N * kPB;                   // rows (i, k): i * b1 + k
  bf16* Ys = Kt + N * kPB;
  float* Qt = reinterpret_cast<float*>(Ys + N * kPB);  // rows (k, i): k * b2 + i
  float* Hs = Qt + N * kPF;                  // (i, k)
  float* W = Hs + N;                         // L rows (i, l), kMaxB weights each
  const long g = blockIdx.x;
  const int tid = threadIdx.x;
  // kParts consecutive threads share a row; each takes kChunks of its 8-column chunks
  const int row = tid / kParts, part = tid % kParts;
  const int c0 = part * kChunks;
  const unsigned mask = 0xffffffffu;

  // q, k, v of the head into shared memory (16-byte chunks)
  {
    const uint4* gq = reinterpret_cast<const uint4*>(q + g * N * kD);
    const uint4* gk = reinterpret_cast<const uint4*>(k + g * N * kD);
    const uint4* gv = reinterpret_cast<const uint4*>(v + g * N * kD);
    for (int x = tid; x < N * (kD / 8); x += kThreads) {
      const int r = x / (kD / 8), c = x % (kD / 8);
      const int so = r * kPB + c * 8;
      *reinterpret_cast<uint4*>(Qs + so) = __ldg(gq + x);
      *reinterpret_cast<uint4*>(Ks + so) = __ldg(gk + x);
      *reinterpret_cast<uint4*>(Vs + so) = __ldg(gv + x);
    }
  }
  __syncthreads();
  const bool active = row < N;
  // step-one aggregated queries (uniform L): row (k, i) gets mean_l q_(l,i)
  if (active) {
    const int i = row % b2;
    float* dst = Qt + row * kPF;
    const float inv = 1.f / (float)b1;
#pragma unroll
    for (int c = c0; c < c0 + kChunks; ++c) {
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      for (int l = 0; l < b1; ++l) {
        float x[8];
        unpack8(*reinterpret_cast<const uint4*>(Qs + (l * b2 + i) * kPB + c * 8), x);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] += x[e];
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) dst[c * 8 + e] = acc[e] * inv;
    }
  }
  __syncthreads();

  for (int t = 1; t <= T; ++t) {
    const bool last = t == T;
    // ---- R-update: row (k, i) ----
    {
      const int kk = row / b2, i = row % b2;
      const float* qt = Qt + (active ? row : 0) * kPF;
      const bf16* kr = Ks + (active ? kk * b2 : 0) * kPB;  // rows of chunk k
      const bf16* vr = Vs + (active ? kk * b2 : 0) * kPB;
      float s[kMaxB];
#pragma unroll
      for (int j = 0; j < kMaxB; ++j) s[j] = 0.f;
      if (active) {
#pragma unroll
        for (int c = c0; c < c0 + kChunks; ++c) {
          const float4 a0 = *reinterpret_cast<const float4*>(qt + c * 8);
          const float4 a1 = *reinterpret_cast<const float4*>(qt + c * 8 + 4);
          const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
#pragma unroll
          for (int j = 0; j < kMaxB; ++j) {
            if (j < b2) {
              float x[8];
              unpack8(*reinterpret_cast<const uint4*>(kr + j * kPB + c * 8), x);
#pragma unroll
              for (int e = 0; e < 8; ++e) s[j] = fmaf(a[e], x[e], s[j]);
            }
          }
        }
      }
      // combine the parts' partial dots (every thread of the row gets the sums)
#pragma unroll
      for (int j = 0; j < kMaxB; ++j) {
#pragma unroll
        for (int o = 1; o < kParts; o <<= 1) s[j] += __shfl_xor_sync(mask, s[j], o);
        s[j] *= sc;
      }
      if (active) {
        float raw[kMaxB];
#pragma unroll
        for (int j = 0; j < kMaxB; ++j) raw[j] = s[j];
        float m;
        const float z = softmax16(s, b2, &m);
        float logit_dot = 0.f;  // sum_j e_j (s_j - m), before normalising
#pragma unroll
        for (int j = 0; j < kMaxB; ++j)
          if (j < b2) logit_dot += s[j] * (raw[j] - m);
        const float inv = 1.f / z;
        if (part == 0) Hs[i * b1 + kk] = __logf(z) - logit_dot * inv;
#pragma unroll
        for (int j = 0; j < kMaxB; ++j) s[j] *= inv;  // R row
        bf16* kt_row = Kt + (i * b1 + kk) * kPB;
        bf16* y_row = Ys + (i * b1 + kk) * kPB;
#pragma unroll
        for (int c = c0; c < c0 + kChunks; ++c) {
          float ak[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
          float av[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int j = 0; j < kMaxB; ++j) {
            if (j < b2) {
              float x[8];
              unpack8(*reinterpret_cast<const uint4*>(kr + j * kPB + c * 8), x);
#pragma unroll
              for (int e = 0; e < 8; ++e) ak[e] = fmaf(s[j], x[e], ak[e]);
              if (last) {
                unpack8(*reinterpret_cast<const uint4*>(vr + j * kPB + c * 8), x);
#pragma unroll
                for (int e = 0; e < 8; ++e) av[e] = fmaf(s[j], x[e], av[e]);
              }
            }
          }
          *reinterpret_cast<uint4*>(kt_row + c * 8) = pack8(ak);
          if (last) *reinterpret_cast<uint4*>(y_row + c * 8) = pack8(av);
        }
      }
    }
    __syncthreads();
    // ---- L-update: row (i, l) ----
    const int ti = row / b1, tl = row % b1;
    float L[kMaxB];
#pragma unroll
    for (int kk = 0; kk < kMaxB; ++kk) L[kk] = 0.f;
    if (active) {
      const bf16* qr = Qs + (tl * b2 + ti) * kPB;
      const bf16* kt = Kt + ti * b1 * kPB;
#pragma unroll
      for (int c = c0; c < c0 + kChunks; ++c) {
        float a[8];
        unpack8(*reinterpret_cast<const uint4*>(qr + c * 8), a);
#pragma unroll
        for (int kk = 0; kk < kMaxB; ++kk) {
          if (kk < b1) {
            float x[8];
            unpack8(*reinterpret_cast<const uint4*>(kt + kk * kPB + c * 8), x);
#pragma unroll
            for (int e = 0; e < 8; ++e) L[kk] = fmaf(a[e], x[e], L[kk]);
          }
        }
      }
    }
#pragma unroll
    for (int kk = 0; kk < kMaxB; ++kk) {
#pragma unroll
      for (int o = 1; o < kParts; o <<= 1) L[kk] += __shfl_xor_sync(mask, L[kk], o);
    }
    if (active) {
#pragma unroll
      for (int kk = 0; kk < kMaxB; ++kk)
        L[kk] = kk < b1 ? fmaf(L[kk], sc, Hs[ti * b1 + kk]) : 0.f;
      float m;
      const float inv = 1.f / softmax16(L, b1, &m);
#pragma unroll
      for (int kk = 0; kk < kMaxB; ++kk) L[kk] *= inv;
    }
    if (!last) {
      if (active && part == 0) {
#pragma unroll
        for (int kk = 0; kk < kMaxB; ++kk) W[row * kMaxB + kk] = L[kk];
      }
      __syncthreads();
      // aggregation for the next R-update: row (k, i)
      if (active) {
        const int kk = row / b2, i = row % b2;
        float csum = 0.f;
        for (int l = 0; l < b1; ++l) csum += W[(i * b1 + l) * kMaxB + kk];
        const float inv = csum > 0.f ? 1.f / csum : 0.f;  // c = 0: Qt := 0
        float* dst = Qt + row * kPF;
#pragma unroll
        for (int c = c0; c < c0 + kChunks; ++c) {
          float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
          for (int l = 0; l < b1; ++l) {
            const float wl = W[(i * b1 + l) * kMaxB + kk];
            float x[8];
            unpack8(*reinterpret_cast<const uint4*>(Qs + (l * b2 + i) * kPB + c * 8), x);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] = fmaf(wl, x[e], acc[e]);
          }
#pragma unroll
          for (int e = 0; e < 8; ++e) dst[c * 8 + e] = acc[e] * inv;
        }
      }
      __syncthreads();
    } else if (active) {
      // output row (l, i) = sum_k L_k Y_{i,k}
      const bf16* yr = Ys + ti * b1 * kPB;
      uint4* orow = reinterpret_cast<uint4*>(out + (g * N + tl * b2 + ti) * kD);
#pragma unroll
      for (int c = c0; c < c0 + kChunks; ++c) {
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int kk = 0; kk < kMaxB; ++kk) {
          if (kk < b1) {
            float x[8];
            unpack8(*reinterpret_cast<const uint4*>(yr + kk * kPB + c * 8), x);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] = fmaf(L[kk], x[e], acc[e]);
          }
        }
        orow[c] = pack8(acc);
      }
    }
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
