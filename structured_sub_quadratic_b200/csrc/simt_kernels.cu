// SIMT kernels for the MonarchAttention forward pass: the general path.
//
// They handle every shape the C ABI accepts (any b1, b2, c1, c2, T, d <= 256)
// in fp32 arithmetic, for fp32 or bf16 inputs, with fp32 intermediates.  The
// float32 entry point runs on them; the bf16 entry point uses them for the
// shapes the tensor-core kernels do not take.  One warp owns one softmax row
// and keeps a running (max, sum) so that rows of any length stream through.
//
// Steps (MonarchAttention OpenReview discussion, eq. (6) objective and the
// alternating maximisation; MonarchRT summary, "Method" (1)-(3)):
//   init      Qt0_{p,i}  = mean_{l in p} q_(l,i)                  (uniform L)
//   R-update  R_{k,p}[i, j in q] = softmax_j(sc Qt_{k,p,q,i} . k_(k,j))
//             Kt = sum R k,  Y = sum R v,  Hs = entropy of that R row
//   L-update  L_i[l,(k,q)] = softmax_(k,q)(sc q_(l,i).Kt_{k,p(l),q,i} + Hs_{k,p(l),q,i})
//             non-final: Qt_{k,p,q,i} = sum_{l in p} L q_(l,i) / sum_{l in p} L
//             final:     O_(l,i) = sum_(k,q) L Y_{k,p(l),q,i}
//
// Workspace layouts (fp32 unless noted; Kt and Y are fp32 or bf16, TW):
//   Qt0 [G][c1][b2][d]           Qt [G][b1 k][c1][c2][b2][d]
//   Kt, Y [G][b2 i][c1 p][b1 k][c2 q][d]   Hs [G][b2][c1][b1][c2]
//   lse [G][b2 i][b1 l]          Ybar [G][d]
// Kt/Y/Hs are position-major so that the (k, q) keys of one (i, p) are
// contiguous for the L-side.
#include "simt_kernels.cuh"
#include "timing.cuh"

#include <math.h>

#include <type_traits>

namespace monarch {

namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;

template <typename TIn>
__global__ void init_qt_kernel(const TIn* __restrict__ Q, float* __restrict__ qt0, Problem pb) {
  const long tid = blockIdx.x * (long)blockDim.x + threadIdx.x;
  const long total = (long)pb.G * pb.c1 * pb.b2 * pb.d;
  if (tid >= total) return;
  const int x = (int)(tid % pb.d);
  long r = tid / pb.d;
  const int i = (int)(r % pb.b2);
  r /= pb.b2;
  const int p = (int)(r % pb.c1);
  const long g = r / pb.c1;
  int l0 = group_start(pb.b1, pb.c1, p), l1 = group_start(pb.b1, pb.c1, p + 1);
  real_rows(pb, i, l0, l1, &l0, &l1);  // the group's real rows at position i
  const TIn* base = Q + (g * pb.b1 * pb.b2 + i) * (long)pb.d + x;
  float s = 0.f;
  for (int l = l0; l < l1; ++l) s += to_f32(base[(long)l * pb.b2 * pb.d]);
  qt0[tid] = l1 > l0 ? s / (float)(l1 - l0) : 0.f;
}

// One block per (g, k); one warp per R row (p, q, i).
template <typename TIn, typename TW, int DV>
__global__ void __launch_bounds__(kThreads)
r_update_kernel(const TIn* __restrict__ K, const TIn* __restrict__ V,
                const float* __restrict__ qt, QtStrides st, TW* __restrict__ kt,
                TW* __restrict__ y, float* __restrict__ hs, Problem pb, int write_y) {
  extern __shared__ float smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int d = pb.d, b1 = pb.b1, b2 = pb.b2, c1 = pb.c1, c2 = pb.c2;
  const int k = (int)(blockIdx.x % b1);
  const long g = blockIdx.x / b1;
  float* sq = smem + warp * d;
  const TIn* Kk = K + (g * b1 + k) * (long)b2 * d;
  const TIn* Vk = V + (g * b1 + k) * (long)b2 * d;
  const int nrows = c1 * c2 * b2;
  for (int r = warp; r < nrows; r += kWarps) {
    const int i = r % b2, q = (r / b2) % c2, p = r / (b2 * c2);
    const float* qv = qt + g * st.g + k * st.k + p * st.p + q * st.q + i * st.i;
    for (int x = lane; x < d; x += 32) sq[x] = qv[x] * pb.sc;
    __syncwarp();
    const int j0 = group_start(b2, c2, q), j1 = group_start(b2, c2, q + 1);
    float m = -INFINITY, z = 0.f, t = 0.f;  // t = sum_j e_j (s_j - m)
    float ak[DV], av[DV];
#pragma unroll
    for (int u = 0; u < DV; ++u) ak[u] = av[u] = 0.f;
    for (int jb = j0; jb < j1; jb += 32) {
      const int j = jb + lane;
      const bool valid = j < j1 && is_real(pb, (long)k * b2 + j);  // pad keys: zero weight
      const float s = valid ? dot_row(sq, Kk + (long)j * d, d) : -INFINITY;
      const float mn = fmaxf(m, warp_max(s));
      const float alpha = (m == -INFINITY) ? 0.f : expf(m - mn);
      const float e = valid ? expf(s - mn) : 0.f;  // valid implies mn finite
      t = (m == -INFINITY) ? 0.f : alpha * (t + z * (m - mn));
      z = z * alpha + warp_sum(e);
      t += warp_sum(valid ? e * (s - mn) : 0.f);
#pragma unroll
      for (int u = 0; u < DV; ++u) { ak[u] *= alpha; av[u] *= alpha; }
      const int nj = min(32, j1 - jb);
      for (int jj = 0; jj < nj; ++jj) {
        const float ej = __shfl_sync(0xffffffffu, e, jj);
        const TIn* kr = Kk + (long)(jb + jj) * d;
        const TIn* vr = Vk + (long)(jb + jj) * d;
#pragma unroll
        for (int u = 0; u < DV; ++u) {
          const int x = lane + 32 * u;
          if (x < d) {
            ak[u] = fmaf(ej, to_f32(kr[x]), ak[u]);
            if (write_y) av[u] = fmaf(ej, to_f32(vr[x]), av[u]);
          }
        }
      }
      m = mn;
    }
    // a group without a real key: Kt = Y = 0 and an entropy bias of -inf,
    // which gives it zero weight in the L-update
    const float inv = z > 0.f ? 1.f / z : 0.f;
    const long orow = (((g * b2 + i) * c1 + p) * b1 + k) * (long)c2 + q;
#pragma unroll
    for (int u = 0; u < DV; ++u) {
      const int x = lane + 32 * u;
      if (x < d) {
        kt[orow * d + x] = from_f32<TW>(ak[u] * inv);
        if (write_y) y[orow * d + x] = from_f32<TW>(av[u] * inv);
      }
    }
    if (lane == 0) hs[orow] = z > 0.f ? logf(z) - t * inv : -INFINITY;
    __syncwarp();
  }
}

// One warp per query row (g, i, l).  MODE 0 writes O, MODE 1 writes the
// row's log-sum-exp (used by the aggregation of a non-final L-update).
template <typename TIn, typename TW, int DV, int MODE>
__global__ void __launch_bounds__(kThreads)
l_rows_kernel(const TIn* __restrict__ Q, const TW* __restrict__ kt,
              const TW* __restrict__ y, const float* __restrict__ hs, TIn* __restrict__ O,
              float* __restrict__ lse, Problem pb) {
  extern __shared__ float smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int d = pb.d, b1 = pb.b1, b2 = pb.b2, c1 = pb.c1, c2 = pb.c2;
  const int nlb = (b1 + kWarps - 1) / kWarps;
  const int lb = (int)(blockIdx.x % nlb);
  const long r = blockIdx.x / nlb;
  const int i = (int)(r % b2);
  const long g = r / b2;
  const int l = lb * kWarps + warp;
  if (l >= b1) return;
  if (!is_real(pb, (long)l * b2 + i)) return;  // pad query rows: no output, no statistics
  const int p = group_of(b1, c1, l);
  float* sq = smem + warp * d;
  const TIn* qrow = Q + ((g * b1 + l) * b2 + i) * (long)d;
  for (int x = lane; x < d; x += 32) sq[x] = to_f32(qrow[x]) * pb.sc;
  __syncwarp();
  const int nk = b1 * c2;
  const long kbase = ((g * b2 + i) * c1 + p) * (long)nk;
  float m = -INFINITY, z = 0.f;
  float ao[DV];
#pragma unroll
  for (int u = 0; u < DV; ++u) ao[u] = 0.f;
  for (int kb = 0; kb < nk; kb += 32) {
    const int kk = kb + lane;
    const bool valid = kk < nk;
    const float s = valid ? dot_row(sq, kt + (kbase + kk) * d, d) + hs[kbase + kk] : -INFINITY;
    const float mn = fmaxf(m, warp_max(s));
    const float alpha = (m == -INFINITY) ? 0.f : expf(m - mn);
    // keys of a group without a real key have s = -inf (so does a whole block of them)
    const float e = s > -INFINITY ? expf(s - mn) : 0.f;
    z = z * alpha + warp_sum(e);
    if (MODE == 0) {
#pragma unroll
      for (int u = 0; u < DV; ++u) ao[u] *= alpha;
      const int nj = min(32, nk - kb);
      for (int jj = 0; jj < nj; ++jj) {
        const float ej = __shfl_sync(0xffffffffu, e, jj);
        const TW* yr = y + (kbase + kb + jj) * d;
#pragma unroll
        for (int u = 0; u < DV; ++u) {
          const int x = lane + 32 * u;
          if (x < d) ao[u] = fmaf(ej, to_f32(yr[x]), ao[u]);
        }
      }
    }
    m = mn;
  }
  if (MODE == 0) {
    const float inv = 1.f / z;
    TIn* orow = O + ((g * b1 + l) * b2 + i) * (long)d;
#pragma unroll
    for (int u = 0; u < DV; ++u) {
      const int x = lane + 32 * u;
      if (x < d) orow[x] = from_f32<TIn>(ao[u] * inv);
    }
  } else {
    if (lane == 0) lse[(g * b2 + i) * b1 + l] = m + logf(z);
  }
}

// Non-final L-update, aggregation side: one warp per key (g, i, p, k, q)
// sums the normalised L column over the rows l of group p.
template <typename TIn, typename TW, int DV>
__global__ void __launch_bounds__(kThreads)
l_aggregate_kernel(const TIn* __restrict__ Q, const TW* __restrict__ kt,
                   const float* __restrict__ hs, const float* __restrict__ lse,
                   float* __restrict__ qt, Problem pb) {
  extern __shared__ float smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int d = pb.d, b1 = pb.b1, b2 = pb.b2, c1 = pb.c1, c2 = pb.c2;
  const int nk = b1 * c2;
  const int nkb = (nk + kWarps - 1) / kWarps;
  const int kb = (int)(blockIdx.x % nkb);
  long r = blockIdx.x / nkb;
  const int p = (int)(r % c1);
  r /= c1;
  const int i = (int)(r % b2);
  const long g = r / b2;
  const int kk = kb * kWarps + warp;
  if (kk >= nk) return;
  const int k = kk / c2, q = kk % c2;
  const long key = ((g * b2 + i) * c1 + p) * (long)nk + kk;
  float* sk = smem + warp * d;
  for (int x = lane; x < d; x += 32) sk[x] = to_f32(kt[key * d + x]) * pb.sc;
  __syncwarp();
  const float bias = hs[key];
  const int l0 = group_start(b1, c1, p), l1 = group_start(b1, c1, p + 1);
  const float* lse_i = lse + (g * b2 + i) * (long)b1;
  float c = 0.f;
  float acc[DV];
#pragma unroll
  for (int u = 0; u < DV; ++u) acc[u] = 0.f;
  for (int lb = l0; lb < l1; lb += 32) {
    const int l = lb + lane;
    const bool valid = l < l1 && is_real(pb, (long)l * b2 + i);  // pad rows: zero weight
    float P = 0.f;
    if (valid) {
      const float s = dot_row(sk, Q + ((g * b1 + l) * b2 + i) * (long)d, d) + bias - lse_i[l];
      P = expf(s);
    }
    c += warp_sum(P);
    const int nl = min(32, l1 - lb);
    for (int jj = 0; jj < nl; ++jj) {
      const float pj = __shfl_sync(0xffffffffu, P, jj);
      const TIn* qrow = Q + ((g * b1 + lb + jj) * b2 + i) * (long)d;
#pragma unroll
      for (int u = 0; u < DV; ++u) {
        const int x = lane + 32 * u;
        if (x < d) acc[u] = fmaf(pj, to_f32(qrow[x]), acc[u]);
      }
    }
  }
  float* out = qt + ((((g * b1 + k) * c1 + p) * c2 + q) * (long)b2 + i) * d;
  const float inv = c > 0.f ? 1.f / c : 0.f;
#pragma unroll
  for (int u = 0; u < DV; ++u) {
    const int x = lane + 32 * u;
    if (x < d) out[x] = acc[u] * inv;
  }
}

// T = 0: every row of M is the uniform Monarch row, so O is the same for all
// tokens of a head: sum over (k, q) of mean_{j in q} v_(k,j) / (b1 c2).
// With padding, the means run over the real keys and the groups with at
// least one real key.
template <typename TIn>
__global__ void ybar_kernel(const TIn* __restrict__ V, float* __restrict__ ybar, Problem pb) {
  const long g = blockIdx.x;
  const int d = pb.d, b1 = pb.b1, b2 = pb.b2, c2 = pb.c2;
  for (int x = threadIdx.x; x < d; x += blockDim.x) {
    float acc = 0.f;
    int groups_used = 0;
    for (int k = 0; k < b1; ++k) {
      for (int q = 0; q < c2; ++q) {
        const int j0 = group_start(b2, c2, q), j1 = group_start(b2, c2, q + 1);
        float s = 0.f;
        int n = 0;
        for (int j = j0; j < j1; ++j) {
          if (!is_real(pb, (long)k * b2 + j)) continue;
          s += to_f32(V[((g * b1 + k) * b2 + j) * (long)d + x]);
          ++n;
        }
        if (n > 0) {
          acc += s / (float)n;
          ++groups_used;
        }
      }
    }
    ybar[g * d + x] = acc / (float)groups_used;
  }
}

template <typename TIn>
__global__ void broadcast_kernel(const float* __restrict__ ybar, TIn* __restrict__ O, Problem pb) {
  const long N = (long)pb.b1 * pb.b2;
  const long total = (long)pb.G * N * pb.d;
  for (long e = blockIdx.x * (long)blockDim.x + threadIdx.x; e < total;
       e += (long)gridDim.x * blockDim.x) {
    const int x = (int)(e % pb.d);
    const long g = e / (N * pb.d);
    O[e] = from_f32<TIn>(ybar[g * pb.d + x]);
  }
}

inline unsigned blocks_for(long n, int threads) { return (unsigned)((n + threads - 1) / threads); }

template <typename TIn, typename TW, int DV>
cudaError_t run(const TIn* q, const TIn* k, const TIn* v, TIn* out, const Problem& pb,
                const SimtWorkspace& ws, cudaStream_t stream, int* launches, bool final_output) {
  TW* kt = static_cast<TW*>(ws.kt);
  TW* yw = static_cast<TW*>(ws.y);
  const int G = pb.G, b1 = pb.b1, b2 = pb.b2, c1 = pb.c1, c2 = pb.c2, d = pb.d;
  const size_t shm = (size_t)kWarps * d * sizeof(float);
  cudaError_t err;
#define MONARCH_LAUNCH(name, ...)                                                     \
  do {                                                                                \
    err = timed_launch(name, stream, launches, [&] { __VA_ARGS__; });                 \
    if (err != cudaSuccess) return err;                                               \
  } while (0)
  if (pb.T == 0) {
    MONARCH_LAUNCH("simt_ybar", (ybar_kernel<TIn><<<G, 128, 0, stream>>>(v, ws.ybar, pb)));
    const long total = (long)G * b1 * b2 * d;
    const unsigned nb = (unsigned)std::min<long>(blocks_for(total, 256), 148L * 16);
    MONARCH_LAUNCH("simt_broadcast",
                   (broadcast_kernel<TIn><<<nb, 256, 0, stream>>>(ws.ybar, out, pb)));
    return cudaSuccess;
  }
  MONARCH_LAUNCH("simt_init_qt",
                 (init_qt_kernel<TIn><<<blocks_for((long)G * c1 * b2 * d, 256), 256, 0, stream>>>(
                     q, ws.qt0, pb)));
  const QtStrides s0 = {(long)c1 * b2 * d, 0, (long)b2 * d, 0, (long)d};
  const QtStrides s1 = {(long)b1 * c1 * c2 * b2 * d, (long)c1 * c2 * b2 * d, (long)c2 * b2 * d,
                        (long)b2 * d, (long)d};
  for (int t = 1; t <= pb.T; ++t) {
    const bool last = (t == pb.T);
    MONARCH_LAUNCH("simt_r_update",
                   (r_update_kernel<TIn, TW, DV><<<(unsigned)((long)G * b1), kThreads, shm,
                                                   stream>>>(k, v, t == 1 ? ws.qt0 : ws.qt,
                                                             t == 1 ? s0 : s1, kt, yw, ws.hs, pb,
                                                             last ? 1 : 0)));
    const unsigned nrow_blocks = (unsigned)((long)G * b2 * ((b1 + kWarps - 1) / kWarps));
    if (last) {
      if (final_output)
        MONARCH_LAUNCH("simt_l_output",
                       (l_rows_kernel<TIn, TW, DV, 0><<<nrow_blocks, kThreads, shm, stream>>>(
                           q, kt, yw, ws.hs, out, nullptr, pb)));
    } else {
      MONARCH_LAUNCH("simt_l_stats",
                     (l_rows_kernel<TIn, TW, DV, 1><<<nrow_blocks, kThreads, shm, stream>>>(
                         q, kt, yw, ws.hs, nullptr, ws.lse, pb)));
      const unsigned nagg = (unsigned)((long)G * b2 * c1 * ((b1 * c2 + kWarps - 1) / kWarps));
      MONARCH_LAUNCH("simt_l_aggregate",
                     (l_aggregate_kernel<TIn, TW, DV><<<nagg, kThreads, shm, stream>>>(
                         q, kt, ws.hs, ws.lse, ws.qt, pb)));
    }
  }
#undef MONARCH_LAUNCH
  return cudaSuccess;
}

}  // namespace

SimtWorkspaceSizes simt_workspace_sizes(const Problem& pb) {
  SimtWorkspaceSizes s;
  const size_t G = pb.G, b1 = pb.b1, b2 = pb.b2, c1 = pb.c1, c2 = pb.c2, d = pb.d;
  s.qt0 = pb.T >= 1 ? G * c1 * b2 * d : 0;
  s.qt = pb.T >= 2 ? G * b1 * c1 * c2 * b2 * d : 0;
  s.kt = pb.T >= 1 ? G * b2 * c1 * b1 * c2 * d : 0;
  s.y = s.kt;
  s.hs = pb.T >= 1 ? G * b2 * c1 * b1 * c2 : 0;
  s.lse = pb.T >= 2 ? G * b2 * b1 : 0;
  s.ybar = pb.T == 0 ? G * d : 0;
  return s;
}

template <typename TIn, typename TW>
cudaError_t simt_r_update(const TIn* k, const TIn* v, const float* qt, const QtStrides& st,
                          TW* kt, TW* y, float* hs, const Problem& pb, bool write_y,
                          cudaStream_t stream, int* launches) {
  const size_t shm = (size_t)kWarps * pb.d * sizeof(float);
  const unsigned nb = (unsigned)((long)pb.G * pb.b1);
  auto go = [&](auto dv) {
    constexpr int DV = decltype(dv)::value;
    return timed_launch("simt_r_update", stream, launches, [&] {
      r_update_kernel<TIn, TW, DV><<<nb, kThreads, shm, stream>>>(k, v, qt, st, kt, y, hs, pb,
                                                                  write_y ? 1 : 0);
    });
  };
  if (pb.d <= 32) return go(std::integral_constant<int, 1>());
  if (pb.d <= 64) return go(std::integral_constant<int, 2>());
  if (pb.d <= 128) return go(std::integral_constant<int, 4>());
  return go(std::integral_constant<int, 8>());
}

template <typename TIn, typename TW>
cudaError_t simt_l_update(const TIn* q, const TW* kt, const float* hs, float* lse, float* qt,
                          const Problem& pb, cudaStream_t stream, int* launches) {
  const size_t shm = (size_t)kWarps * pb.d * sizeof(float);
  const int G = pb.G, b1 = pb.b1, b2 = pb.b2, c1 = pb.c1, c2 = pb.c2;
  const unsigned nrow_blocks = (unsigned)((long)G * b2 * ((b1 + kWarps - 1) / kWarps));
  const unsigned nagg = (unsigned)((long)G * b2 * c1 * ((b1 * c2 + kWarps - 1) / kWarps));
  auto go = [&](auto dv) {
    constexpr int DV = decltype(dv)::value;
    cudaError_t e = timed_launch("simt_l_stats", stream, launches, [&] {
      l_rows_kernel<TIn, TW, DV, 1><<<nrow_blocks, kThreads, shm, stream>>>(
          q, kt, (const TW*)nullptr, hs, (TIn*)nullptr, lse, pb);
    });
    if (e != cudaSuccess) return e;
    return timed_launch("simt_l_aggregate", stream, launches, [&] {
      l_aggregate_kernel<TIn, TW, DV><<<nagg, kThreads, shm, stream>>>(q, kt, hs, lse, qt, pb);
    });
  };
  if (pb.d <= 32) return go(std::integral_constant<int, 1>());
  if (pb.d <= 64) return go(std::integral_constant<int, 2>());
  if (pb.d <= 128) return go(std::integral_constant<int, 4>());
  return go(std::integral_constant<int, 8>());
}

template cudaError_t simt_r_update<bf16, bf16>(const bf16*, const bf16*, const float*,
                                               const QtStrides&, bf16*, bf16*, float*,
                                               const Problem&, bool, cudaStream_t, int*);
template cudaError_t simt_l_update<bf16, bf16>(const bf16*, const bf16*, const float*, float*,
                                               float*, const Problem&, cudaStream_t, int*);

template <typename TIn, typename TW>
cudaError_t simt_forward(const TIn* q, const TIn* k, const TIn* v, TIn* out, const Problem& pb,
                         const SimtWorkspace& ws, cudaStream_t stream, int* launches,
                         bool final_output) {
  if (pb.d <= 32) return run<TIn, TW, 1>(q, k, v, out, pb, ws, stream, launches, final_output);
  if (pb.d <= 64) return run<TIn, TW, 2>(q, k, v, out, pb, ws, stream, launches, final_output);
  if (pb.d <= 128) return run<TIn, TW, 4>(q, k, v, out, pb, ws, stream, launches, final_output);
  return run<TIn, TW, 8>(q, k, v, out, pb, ws, stream, launches, final_output);
}

#define MONARCH_INSTANTIATE(TIn, TW)                                                        \
  template cudaError_t simt_forward<TIn, TW>(const TIn*, const TIn*, const TIn*, TIn*,      \
                                             const Problem&, const SimtWorkspace&,          \
                                             cudaStream_t, int*, bool);
MONARCH_INSTANTIATE(float, float)
MONARCH_INSTANTIATE(bf16, float)
MONARCH_INSTANTIATE(bf16, bf16)
#undef MONARCH_INSTANTIATE

}  // namespace monarch
