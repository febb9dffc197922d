// CUDA-core kernels for shapes whose groups are too small for the tcgen05
// tiles.  The video layouts (hw,f) and (f,hw) of a latent with three frames
// have column groups of 3 keys over 3 positions, or rows of 3 keys: a
// 128-row tensor-core tile would hold 3 to 6 real rows and a 16-key column
// tile 3 real keys, so those kernels spend their time on empty tiles.  The
// work per group is then a few 128-element dot products, and the pass is
// bound by reading q, k, v, Kt and Y once.  Here one warp owns a group; each
// lane holds d/32 consecutive elements of every row it touches (8-byte loads
// and stores, a whole row per warp instruction), dot products are finished
// with a butterfly of shuffles (every lane ends with the same sum, so every
// lane takes the same softmax), and the arithmetic is fp32.  The launches
// are timed as cc_init_qt, cc_r_update and cc_l_output (CUDA cores).
//
// The steps follow the alternating maximisation of MonarchAttention
// (MonarchAttention OpenReview discussion, the R- and L-updates; MonarchRT
// summary, "Method"):
//   aggregation  Qt0_{p,i} = mean over the rows l of group p of q_(l,i)
//   R-update     R = softmax over the keys j of group q of Qt.K_j / sqrt(d),
//                Kt = R K, Y = R V, Hs = entropy of R
//   output       L = softmax over the keys (k, q) of q.Kt / sqrt(d) + Hs,
//                O = L Y
#include "small_dim.cuh"

#include <cooperative_groups.h>
#include <math.h>

#include "launch.cuh"
#include "tc_ptx.cuh"
#include "timing.cuh"

namespace monarch {

namespace {

using namespace tc;

constexpr int kMaxKeys = 8;   // keys per R-update group or per output row
constexpr int kMaxPos = 32;   // positions per chunk in the R-update
constexpr int kMaxRows = 16;  // rows per group in the aggregation
constexpr int kWarps = 8;     // warps per block
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.69314718055994531f;

// E consecutive bf16 elements of a row <-> fp32 registers (E = d / 32).
template <int E>
__device__ __forceinline__ void load_row(const bf16* p, float (&x)[E]) {
  static_assert(E == 2 || E == 4, "d = 64 or 128");
  if constexpr (E == 4) {
    const uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
    x[0] = __uint_as_float(u.x << 16);
    x[1] = __uint_as_float(u.x & 0xffff0000u);
    x[2] = __uint_as_float(u.y << 16);
    x[3] = __uint_as_float(u.y & 0xffff0000u);
  } else {
    const uint32_t u = __ldg(reinterpret_cast<const unsigned int*>(p));
    x[0] = __uint_as_float(u << 16);
    x[1] = __uint_as_float(u & 0xffff0000u);
  }
}

template <int E>
__device__ __forceinline__ void store_row(bf16* p, const float (&x)[E]) {
  if constexpr (E == 4) {
    *reinterpret_cast<uint2*>(p) = make_uint2(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]));
  } else {
    *reinterpret_cast<uint32_t*>(p) = pack_bf16x2(x[0], x[1]);
  }
}

// Sum over the warp; every lane receives the same value (each butterfly
// step adds the same two operands on both partners).
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

template <int E>
__device__ __forceinline__ float dot_part(const float (&a)[E], const float (&b)[E]) {
  float s = a[0] * b[0];
#pragma unroll
  for (int e = 1; e < E; ++e) s = fmaf(a[e], b[e], s);
  return s;
}

// Unit (g, p, i) of the aggregation, in Qt0's row order.
template <int D>
__global__ void __launch_bounds__(kWarps * 32)
    small_init_kernel(const bf16* __restrict__ q, bf16* __restrict__ qt0, Problem pb) {
  constexpr int E = D / 32;
  const int lane = threadIdx.x & 31;
  // 32-bit index arithmetic (the launch checks that every index fits)
  const int unit = (int)blockIdx.x * kWarps + (int)(threadIdx.x >> 5);
  // qt0 may still be read by the previous call's R-update
  pdl_wait();
  pdl_launch_dependents();
  if (unit >= pb.G * pb.c1 * pb.b2) return;
  const int i = unit % pb.b2;
  const int gp = unit / pb.b2;
  const int p = gp % pb.c1;
  const int g = gp / pb.c1;
  const int l0 = group_start(pb.b1, pb.c1, p), l1 = group_start(pb.b1, pb.c1, p + 1);
  float acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
  for (int l = l0; l < l1; ++l) {
    float x[E];
    load_row<E>(q + token_row(pb, g, l, i) * D + lane * E, x);
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] += x[e];
  }
  const float n = (float)(l1 - l0);
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] /= n;
  store_row<E>(qt0 + (long)unit * D + lane * E, acc);
}

// Aggregation of a few long row groups (fewer (g, p, i) units than a
// quarter of the SMs, each of >= kSplitMinRows rows): a cluster of kSplit
// CTAs per unit, CTA r summing the r-th slice of the group's rows (16-byte
// column chunks x row lanes, warp shuffles, then the warps in shared
// memory); CTA 0 adds the kSplit slice sums in rank order through
// distributed shared memory, so the result does not depend on scheduling.
constexpr int kSplit = 8;
constexpr int kSplitMinRows = 256;

template <int D>
__global__ void __launch_bounds__(256)
    split_init_kernel(const bf16* __restrict__ q, bf16* __restrict__ qt0, Problem pb) {
  namespace cg = cooperative_groups;
  constexpr int CH = D / 8;     // 16-byte chunks per row
  constexpr int RL = 256 / CH;  // row lanes
  __shared__ float red[8][D];
  __shared__ float part[D];     // this CTA's slice sum, read by CTA 0 of the cluster
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int unit = (int)blockIdx.x / kSplit;  // (g c1 + p) b2 + i
  const int i = unit % pb.b2;
  const int gp = unit / pb.b2;
  const int p = gp % pb.c1;
  const int g = gp / pb.c1;
  const int l0 = group_start(pb.b1, pb.c1, p), l1 = group_start(pb.b1, pb.c1, p + 1);
  const int n = l1 - l0;
  const int s0 = l0 + (int)((long)n * rank / kSplit), s1 = l0 + (int)((long)n * (rank + 1) / kSplit);
  pdl_wait();  // qt0 may still be read by the previous call's R-update
  pdl_launch_dependents();
  const int ch = threadIdx.x % CH, rl = threadIdx.x / CH, lane = threadIdx.x & 31;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  const uint4* base = reinterpret_cast<const uint4*>(q + token_row(pb, g, 0, i) * D) + ch;
  const long row_stride = (pb.tr ? (long)D : (long)pb.b2 * D) / 8;  // rows l apart, in uint4
#pragma unroll 4
  for (int l = s0 + rl; l < s1; l += RL) {
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
    for (int w8 = 0; w8 < 8; ++w8) sum += red[w8][threadIdx.x];
    part[threadIdx.x] = sum;
  }
  cluster.sync();  // every slice sum is in its CTA's shared memory
  if (rank == 0 && threadIdx.x < D) {
    float sum = 0.f;
#pragma unroll
    for (int r = 0; r < kSplit; ++r) sum += cluster.map_shared_rank(part, r)[threadIdx.x];
    qt0[(long)unit * D + threadIdx.x] = __float2bfloat16_rn(sum / (float)n);
  }
  cluster.sync();  // CTA 0 has read every slice sum before any CTA exits
}

// Sub-item (g, p, k, q) of the R-update, in the tensor-core kernels' order;
// NK keys of register space (4 or 8).
template <int D, int NK>
__global__ void __launch_bounds__(kWarps * 32)
    small_r_kernel(const bf16* __restrict__ qt, const bf16* __restrict__ k,
                   const bf16* __restrict__ v, bf16* __restrict__ kt, bf16* __restrict__ y,
                   float* __restrict__ hs, Problem pb, int qt_per_item, int write_y) {
  constexpr int E = D / 32;
  const int lane = threadIdx.x & 31;
  // 32-bit index arithmetic (the launch checks that every index fits)
  const int sub = (int)blockIdx.x * kWarps + (int)(threadIdx.x >> 5);
  pdl_wait();  // the query rows come from the previous kernel
  pdl_launch_dependents();
  if (sub >= pb.G * pb.c1 * pb.b1 * pb.c2) return;
  const int q = sub % pb.c2;
  const int item = sub / pb.c2;
  const int kc = item % pb.b1;
  const int gp = item / pb.b1;
  const int p = gp % pb.c1;
  const int g = gp / pb.c1;
  const int js = group_start(pb.b2, pb.c2, q), nq = group_start(pb.b2, pb.c2, q + 1) - js;
  // the group's keys and values, row j of chunk kc
  float kr[NK][E], vr[NK][E];
#pragma unroll
  for (int j = 0; j < NK; ++j) {
    if (j < nq) {
      const long row = token_row(pb, g, kc, js + j);
      load_row<E>(k + row * D + lane * E, kr[j]);
      load_row<E>(v + row * D + lane * E, vr[j]);
    }
  }
  const float sc_log2 = pb.sc * kLog2e;
  // Qt0 [G][c1][b2][d] (step one) or a later step's Qt [G][b1][c1][c2][b2][d]
  const int qset = qt_per_item ? ((g * pb.b1 + kc) * pb.c1 + p) * pb.c2 + q : gp;
  const bf16* qrows = qt + (long)qset * pb.b2 * D + lane * E;
  float qn[E];
  load_row<E>(qrows, qn);
  for (int i = 0; i < pb.b2; ++i) {
    float qv[E];
#pragma unroll
    for (int e = 0; e < E; ++e) qv[e] = qn[e];
    if (i + 1 < pb.b2) load_row<E>(qrows + (long)(i + 1) * D, qn);  // next position's row
    // logits in log2 units, their maximum, exponentials, sum z and
    // t2 = sum_j e_j (x_j - max) for the entropy
    float s[NK];
    float m = -INFINITY;
#pragma unroll
    for (int j = 0; j < NK; ++j) {
      if (j < nq) {
        s[j] = warp_sum(dot_part<E>(qv, kr[j])) * sc_log2;
        m = fmaxf(m, s[j]);
      }
    }
    float z = 0.f, t2 = 0.f;
#pragma unroll
    for (int j = 0; j < NK; ++j) {
      if (j < nq) {
        const float dd = s[j] - m;
        s[j] = ex2(dd);
        z += s[j];
        t2 = fmaf(s[j], dd, t2);
      }
    }
    const float inv = 1.f / z;
    float ko[E], yo[E];
#pragma unroll
    for (int e = 0; e < E; ++e) ko[e] = yo[e] = 0.f;
#pragma unroll
    for (int j = 0; j < NK; ++j) {
      if (j < nq) {
        const float r = s[j] * inv;
#pragma unroll
        for (int e = 0; e < E; ++e) {
          ko[e] = fmaf(r, kr[j][e], ko[e]);
          yo[e] = fmaf(r, vr[j][e], yo[e]);
        }
      }
    }
    // [G][b2][c1][b1][c2] row of (g, i, p, kc, q)
    const long orow = (long)(((g * pb.b2 + i) * pb.c1 + p) * pb.b1 + kc) * pb.c2 + q;
    store_row<E>(kt + orow * D + lane * E, ko);
    if (write_y) store_row<E>(y + orow * D + lane * E, yo);
    // entropy -sum R ln R = ln z - sum_j e_j (x_j - max) ln 2 / z
    if (lane == 0) hs[orow] = logf(z) - t2 * kLn2 / z;
  }
}

// Item (g, i, p) of the final L-update + output: the |p| rows l of group p
// at position i against the b1 c2 keys (k, q); NK keys of register space.
template <int D, int NK>
__global__ void __launch_bounds__(kWarps * 32)
    small_out_kernel(const bf16* __restrict__ q, const bf16* __restrict__ kt,
                     const bf16* __restrict__ y, const float* __restrict__ hs,
                     bf16* __restrict__ out, Problem pb) {
  constexpr int E = D / 32;
  const int lane = threadIdx.x & 31;
  // 32-bit index arithmetic (the launch checks that every index fits)
  const int item = (int)blockIdx.x * kWarps + (int)(threadIdx.x >> 5);
  pdl_wait();  // Kt, Y and Hs come from the previous kernel
  pdl_launch_dependents();
  if (item >= pb.G * pb.b2 * pb.c1) return;
  const int p = item % pb.c1;
  const int gi = item / pb.c1;
  const int i = gi % pb.b2;
  const int g = gi / pb.b2;
  const int nk = pb.b1 * pb.c2;
  const long key0 = (long)item * nk;  // row ((g b2 + i) c1 + p) nk of Kt, Y and Hs
  float kr[NK][E], yr[NK][E], bias[NK];
#pragma unroll
  for (int j = 0; j < NK; ++j) {
    if (j < nk) {
      load_row<E>(kt + (key0 + j) * D + lane * E, kr[j]);
      load_row<E>(y + (key0 + j) * D + lane * E, yr[j]);
      bias[j] = __ldg(hs + key0 + j);
    }
  }
  const int l0 = group_start(pb.b1, pb.c1, p), l1 = group_start(pb.b1, pb.c1, p + 1);
  float qn[E];
  load_row<E>(q + token_row(pb, g, l0, i) * D + lane * E, qn);
  for (int l = l0; l < l1; ++l) {
    const long row = token_row(pb, g, l, i);
    float qv[E];
#pragma unroll
    for (int e = 0; e < E; ++e) qv[e] = qn[e];
    if (l + 1 < l1) load_row<E>(q + token_row(pb, g, l + 1, i) * D + lane * E, qn);
    float s[NK];
    float m = -INFINITY;
#pragma unroll
    for (int j = 0; j < NK; ++j) {
      if (j < nk) {
        s[j] = fmaf(warp_sum(dot_part<E>(qv, kr[j])), pb.sc, bias[j]);
        m = fmaxf(m, s[j]);
      }
    }
    float z = 0.f;
#pragma unroll
    for (int j = 0; j < NK; ++j) {
      if (j < nk) {
        s[j] = ex2((s[j] - m) * kLog2e);
        z += s[j];
      }
    }
    const float inv = 1.f / z;
    float o[E];
#pragma unroll
    for (int e = 0; e < E; ++e) o[e] = 0.f;
#pragma unroll
    for (int j = 0; j < NK; ++j) {
      if (j < nk) {
        const float w = s[j] * inv;
#pragma unroll
        for (int e = 0; e < E; ++e) o[e] = fmaf(w, yr[j][e], o[e]);
      }
    }
    store_row<E>(out + row * D + lane * E, o);
  }
}

unsigned blocks_for(long warps) { return (unsigned)((warps + kWarps - 1) / kWarps); }

}  // namespace

// The kernels index units, sub-items, items, the query sets of Qt and the
// rows of Kt / Y / Hs ([G][b2][c1][b1][c2]) in 32-bit arithmetic; the largest
// of these counts is G b2 c1 b1 c2.
static bool small_indices_fit(const Problem& pb) {
  return (long)pb.G * pb.b2 * pb.c1 * pb.b1 * pb.c2 < (1L << 31);
}

// A few long row groups: the clustered aggregation (every group of
// >= kSplitMinRows rows, fewer units than a quarter of the SMs).
static bool split_init_fits(const Problem& pb) {
  return (pb.d == 64 || pb.d == 128) && !is_padded(pb) && pb.b1 / pb.c1 >= kSplitMinRows &&
         (long)pb.G * pb.c1 * pb.b2 * 4 < num_sms() && small_indices_fit(pb);
}

bool small_init_fits(const Problem& pb) {
  return ((pb.d == 64 || pb.d == 128) && !is_padded(pb) &&
          (pb.b1 + pb.c1 - 1) / pb.c1 <= kMaxRows && small_indices_fit(pb)) ||
         split_init_fits(pb);
}

bool small_r_fits(const Problem& pb) {
  return (pb.d == 64 || pb.d == 128) && !is_padded(pb) &&
         (pb.b2 + pb.c2 - 1) / pb.c2 <= kMaxKeys && pb.b2 <= kMaxPos && small_indices_fit(pb);
}

bool small_out_fits(const Problem& pb) {
  return (pb.d == 64 || pb.d == 128) && !is_padded(pb) && pb.b1 * pb.c2 <= kMaxKeys &&
         small_indices_fit(pb);
}

cudaError_t launch_small_init(const bf16* q, bf16* qt0, const Problem& pb, cudaStream_t stream,
                              int* launches) {
  if (!small_init_fits(pb)) return cudaErrorInvalidValue;
  if (split_init_fits(pb)) {
    const unsigned units = (unsigned)((long)pb.G * pb.c1 * pb.b2);
    return timed_launch("cc_init_qt", stream, launches, [&] {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(units * kSplit);
      cfg.blockDim = dim3(256);
      cfg.stream = stream;
      cudaLaunchAttribute attr[2];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = kSplit;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      attr[1].val.programmaticStreamSerializationAllowed = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 2;
      return pb.d == 128 ? cudaLaunchKernelEx(&cfg, split_init_kernel<128>, q, qt0, pb)
                         : cudaLaunchKernelEx(&cfg, split_init_kernel<64>, q, qt0, pb);
    });
  }
  const unsigned grid = blocks_for((long)pb.G * pb.c1 * pb.b2);
  return timed_launch("cc_init_qt", stream, launches, [&] {
    return pb.d == 128 ? launch_pdl(small_init_kernel<128>, dim3(grid), dim3(kWarps * 32), 0,
                                    stream, q, qt0, pb)
                       : launch_pdl(small_init_kernel<64>, dim3(grid), dim3(kWarps * 32), 0,
                                    stream, q, qt0, pb);
  });
}

cudaError_t launch_small_r(const bf16* qt, const bf16* k, const bf16* v, bf16* kt, bf16* y,
                           float* hs, const Problem& pb, bool qt_per_item, bool write_y,
                           cudaStream_t stream, int* launches) {
  if (!small_r_fits(pb)) return cudaErrorInvalidValue;
  const unsigned grid = blocks_for((long)pb.G * pb.c1 * pb.b1 * pb.c2);
  const int per_item = qt_per_item ? 1 : 0, wy = write_y ? 1 : 0;
  const bool four = (pb.b2 + pb.c2 - 1) / pb.c2 <= 4;  // fewer registers: more warps per SM
  auto kernel = pb.d == 128 ? (four ? small_r_kernel<128, 4> : small_r_kernel<128, kMaxKeys>)
                            : (four ? small_r_kernel<64, 4> : small_r_kernel<64, kMaxKeys>);
  return timed_launch("cc_r_update", stream, launches, [&] {
    return launch_pdl(kernel, dim3(grid), dim3(kWarps * 32), 0, stream, qt, k, v, kt, y, hs, pb,
                      per_item, wy);
  });
}

cudaError_t launch_small_out(const bf16* q, const bf16* kt, const bf16* y, const float* hs,
                             bf16* out, const Problem& pb, cudaStream_t stream, int* launches) {
  if (!small_out_fits(pb)) return cudaErrorInvalidValue;
  const unsigned grid = blocks_for((long)pb.G * pb.b2 * pb.c1);
  const bool four = pb.b1 * pb.c2 <= 4;
  auto kernel = pb.d == 128 ? (four ? small_out_kernel<128, 4> : small_out_kernel<128, kMaxKeys>)
                            : (four ? small_out_kernel<64, 4> : small_out_kernel<64, kMaxKeys>);
  return timed_launch("cc_l_output", stream, launches, [&] {
    return launch_pdl(kernel, dim3(grid), dim3(kWarps * 32), 0, stream, q, kt, y, hs, out, pb);
  });
}

}  // namespace monarch
