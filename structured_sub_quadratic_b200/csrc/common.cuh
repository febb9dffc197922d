// Device helpers shared by the MonarchAttention kernels.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace monarch {

typedef __nv_bfloat16 bf16;

// ---------------------------------------------------------------------------
// Problem description passed to every launch.  G = B*H independent heads.
// Token n = l*b2 + i.  Row groups p of l in [b1] (c1 of them) and column
// groups q of j in [b2] (c2 of them) are contiguous, sizes differing by at
// most one with the larger groups first.
//
// Padding: a sequence of fewer than b1*b2 tokens sits on the b1*b2 grid with
// its real tokens at [real_lo, real_hi) (pad tokens before and/or after).
// Pad keys get zero R weight, a column group with no real key zero L
// weight (its entropy bias is -inf), and pad query rows are left out of the
// aggregations; unpadded problems have real_lo = 0, real_hi = b1*b2.
// ---------------------------------------------------------------------------
//
// Token order of q, k, v and out: tr = 0 is Monarch order (token l*b2 + i);
// tr = 1 is the transpose (token i*b1 + l), the raster order of a video
// latent in the (w,fh) and (hw,f) layouts.  Intermediates are the same
// either way.
// ---------------------------------------------------------------------------
struct Problem {
  int G, b1, b2, d, T, c1, c2;
  float sc;  // 1/sqrt(d)
  int real_lo, real_hi;
  int tr;
  // Launch-shape hint: when a call is split into groups of heads, the
  // (g, p, i) unit count of the whole call, which the bf16 step-one
  // aggregation's thread count follows (its row sums' order depends on it),
  // so that the split call gives bit-identical results; 0 means G c1 b2.
  long init_units;
};

// Row of token (l, i) of head g in q, k, v and out.
__host__ __device__ __forceinline__ long token_row(const Problem& pb, long g, int l, int i) {
  return pb.tr ? (g * pb.b2 + i) * pb.b1 + l : (g * pb.b1 + l) * pb.b2 + i;
}

__host__ __device__ __forceinline__ bool is_real(const Problem& pb, long m) {
  return m >= pb.real_lo && m < pb.real_hi;
}

__host__ __device__ __forceinline__ bool is_padded(const Problem& pb) {
  return pb.real_lo != 0 || pb.real_hi != pb.b1 * pb.b2;
}

// The rows l in [l0, l1) whose token l*b2 + i is real: [*lr0, *lr1).
__host__ __device__ __forceinline__ void real_rows(const Problem& pb, int i, int l0, int l1,
                                                   int* lr0, int* lr1) {
  const int a = pb.real_lo > i ? (pb.real_lo - i + pb.b2 - 1) / pb.b2 : 0;
  const int b = pb.real_hi > i ? (pb.real_hi - i + pb.b2 - 1) / pb.b2 : 0;
  *lr0 = a > l0 ? a : l0;
  *lr1 = b < l1 ? b : l1;
  if (*lr1 < *lr0) *lr1 = *lr0;
}

__host__ __device__ __forceinline__ int group_start(int n, int c, int g) {
  const int base = n / c, extra = n % c;
  return g * base + (g < extra ? g : extra);
}

__host__ __device__ __forceinline__ int group_of(int n, int c, int x) {
  const int base = n / c, extra = n % c;
  const int cut = extra * (base + 1);
  return x < cut ? x / (base + 1) : extra + (x - cut) / base;
}

// ---------------------------------------------------------------------------
// element conversion
// ---------------------------------------------------------------------------
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(bf16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ bf16 from_f32<bf16>(float x) {
  return __float2bfloat16_rn(x);
}

// ---------------------------------------------------------------------------
// warp reductions
// ---------------------------------------------------------------------------
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// dot(sq[0:d], row[0:d]) where sq is fp32 in shared memory (read as a
// broadcast) and row is one d-long row in global memory.  When d % 8 == 0
// rows are read 16 bytes at a time (rows are 16-byte aligned then).
__device__ __forceinline__ float dot_row(const float* __restrict__ sq,
                                         const float* __restrict__ row, int d) {
  float acc = 0.f;
  if ((d & 3) == 0) {
    const float4* r4 = reinterpret_cast<const float4*>(row);
    for (int x = 0; x < (d >> 2); ++x) {
      const float4 r = __ldg(r4 + x);
      acc = fmaf(sq[4 * x + 0], r.x, acc);
      acc = fmaf(sq[4 * x + 1], r.y, acc);
      acc = fmaf(sq[4 * x + 2], r.z, acc);
      acc = fmaf(sq[4 * x + 3], r.w, acc);
    }
  } else {
    for (int x = 0; x < d; ++x) acc = fmaf(sq[x], __ldg(row + x), acc);
  }
  return acc;
}

__device__ __forceinline__ float dot_row(const float* __restrict__ sq,
                                         const bf16* __restrict__ row, int d) {
  float acc = 0.f;
  if ((d & 7) == 0) {
    const uint4* r8 = reinterpret_cast<const uint4*>(row);
    for (int x = 0; x < (d >> 3); ++x) {
      const uint4 u = __ldg(r8 + x);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const float lo = __uint_as_float(w[t] << 16);
        const float hi = __uint_as_float(w[t] & 0xffff0000u);
        acc = fmaf(sq[8 * x + 2 * t], lo, acc);
        acc = fmaf(sq[8 * x + 2 * t + 1], hi, acc);
      }
    }
  } else {
    for (int x = 0; x < d; ++x) acc = fmaf(sq[x], __bfloat162float(row[x]), acc);
  }
  return acc;
}

// ---------------------------------------------------------------------------
// Device-side status word: kernels with bounded waits record a timeout here
// instead of trapping; the host reads it through monarch_attn_check().
// ---------------------------------------------------------------------------
#define MONARCH_DEVICE_TIMEOUT_FLAG 1

}  // namespace monarch
