// Backward pass of the T = 1 forward (MonarchRT summary, "Method" (3):
// forward and backward kernels for finetuning with one refinement step).
// SIMT kernels in fp32 arithmetic for fp32 or bf16 inputs; every reduction
// runs in a fixed order (no atomics), so results are deterministic.  bf16
// shapes the tensor-core kernels take (bwd_tc.cu) run their recompute, L side
// and (untiled) R side there; the final dq sum always runs here.
//
// Forward quantities are recomputed: Qt0, Kt, Y, Hs by the SIMT forward
// kernels, the L rows' log-sum-exps and O here.  With G = dO:
//   L side, row (l, i):    delta = G . O,  dS_L = L (G . Y - delta),
//                          dq1 = sc sum_{k,q} dS_L Kt
//   L side, key (k,p,q,i): dKt = sc sum_{l in p} dS_L q_(l,i),
//                          dHs = sum dS_L,  dY = sum L G_(l,i)
//   R side, row (k,p,q,i): dR_j = dKt . k_j + dY . v_j - dHs (ln R_j + 1),
//                          dS_R = R (dR - sum_j R dR),
//                          partial dQt0 = sc sum_j dS_R k_j
//   R side, key (k, j):    dk = sum_{p,i} R dKt + sc dS_R Qt0,  dv = sum R dY
//   queries, (p, i):       dQt0 = sum_{k,q} partials,
//                          dq_(l,i) = dq1 + dQt0 / |p|
// Layouts (fp32): Kt, Y, dKt, dY [G][b2 i][c1 p][b1 k][c2 q][d];
// Hs, dHs [G][b2][c1][b1][c2]; lse, delta [G][b2 i][b1 l]; dq1 [G][N][d];
// R, dS_R [G][b1 k][c1 p][b2 i][b2 j]; dQt0 partials [G][c1][b2][b1][c2][d].
#include "bwd_kernels.cuh"

#include <math.h>

#include <type_traits>

#include "bwd_tc.cuh"
#include "simt_kernels.cuh"
#include "timing.cuh"

namespace monarch {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;

// ---- L side, one warp per query row (g, l, i) ----
template <typename TIn, int DV>
__global__ void __launch_bounds__(kThreads)
    l_bwd_rows_kernel(const TIn* __restrict__ Q, const TIn* __restrict__ dO,
                      const float* __restrict__ kt, const float* __restrict__ y,
                      const float* __restrict__ hs, float* __restrict__ dq1,
                      float* __restrict__ lse, float* __restrict__ delta, Problem pb) {
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
  const int p = group_of(b1, c1, l);
  float* sq = smem + warp * 2 * d;
  float* sg = sq + d;
  const long row = (g * b1 + l) * b2 + i;
  for (int x = lane; x < d; x += 32) {
    sq[x] = to_f32(Q[row * d + x]) * pb.sc;
    sg[x] = to_f32(dO[row * d + x]);
  }
  __syncwarp();
  const int nk = b1 * c2;
  const long kbase = ((g * b2 + i) * c1 + p) * (long)nk;
  // pass 1: the row's softmax statistics and O
  float m = -INFINITY, z = 0.f;
  float ao[DV];
#pragma unroll
  for (int u = 0; u < DV; ++u) ao[u] = 0.f;
  for (int kb = 0; kb < nk; kb += 32) {
    const int kk = kb + lane;
    const float s = kk < nk ? dot_row(sq, kt + (kbase + kk) * d, d) + hs[kbase + kk] : -INFINITY;
    const float mn = fmaxf(m, warp_max(s));
    const float alpha = (m == -INFINITY) ? 0.f : expf(m - mn);
    const float e = s > -INFINITY ? expf(s - mn) : 0.f;
    z = z * alpha + warp_sum(e);
#pragma unroll
    for (int u = 0; u < DV; ++u) ao[u] *= alpha;
    const int nj = min(32, nk - kb);
    for (int jj = 0; jj < nj; ++jj) {
      const float ej = __shfl_sync(0xffffffffu, e, jj);
      const float* yr = y + (kbase + kb + jj) * d;
#pragma unroll
      for (int u = 0; u < DV; ++u) {
        const int x = lane + 32 * u;
        if (x < d) ao[u] = fmaf(ej, yr[x], ao[u]);
      }
    }
    m = mn;
  }
  const float lse_row = m + logf(z);
  float dg = 0.f;
#pragma unroll
  for (int u = 0; u < DV; ++u) {
    const int x = lane + 32 * u;
    if (x < d) dg = fmaf(sg[x], ao[u] / z, dg);
  }
  const float delta_row = warp_sum(dg);
  // pass 2: dS_L = L (G . Y - delta); dq1 = sc sum dS_L Kt
  float aq[DV];
#pragma unroll
  for (int u = 0; u < DV; ++u) aq[u] = 0.f;
  for (int kb = 0; kb < nk; kb += 32) {
    const int kk = kb + lane;
    float ds = 0.f;
    if (kk < nk) {
      const float s = dot_row(sq, kt + (kbase + kk) * d, d) + hs[kbase + kk];
      const float Lw = s > -INFINITY ? expf(s - lse_row) : 0.f;
      ds = Lw * (dot_row(sg, y + (kbase + kk) * d, d) - delta_row);
    }
    const int nj = min(32, nk - kb);
    for (int jj = 0; jj < nj; ++jj) {
      const float dj = __shfl_sync(0xffffffffu, ds, jj);
      const float* kr = kt + (kbase + kb + jj) * d;
#pragma unroll
      for (int u = 0; u < DV; ++u) {
        const int x = lane + 32 * u;
        if (x < d) aq[u] = fmaf(dj, kr[x], aq[u]);
      }
    }
  }
#pragma unroll
  for (int u = 0; u < DV; ++u) {
    const int x = lane + 32 * u;
    if (x < d) dq1[row * d + x] = aq[u] * pb.sc;
  }
  if (lane == 0) {
    lse[(g * b2 + i) * b1 + l] = lse_row;
    delta[(g * b2 + i) * b1 + l] = delta_row;
  }
}

// ---- L side, one warp per key (g, i, p, k, q) ----
template <typename TIn, int DV>
__global__ void __launch_bounds__(kThreads)
    l_bwd_keys_kernel(const TIn* __restrict__ Q, const TIn* __restrict__ dO,
                      const float* __restrict__ kt, const float* __restrict__ y,
                      const float* __restrict__ hs, const float* __restrict__ lse,
                      const float* __restrict__ delta, float* __restrict__ dkt,
                      float* __restrict__ dy, float* __restrict__ dhs, Problem pb) {
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
  const long key = ((g * b2 + i) * c1 + p) * (long)nk + kk;
  float* sk = smem + warp * 2 * d;
  float* sy = sk + d;
  for (int x = lane; x < d; x += 32) {
    sk[x] = kt[key * d + x] * pb.sc;
    sy[x] = y[key * d + x];
  }
  __syncwarp();
  const float bias = hs[key];
  const int l0 = group_start(b1, c1, p), l1 = group_start(b1, c1, p + 1);
  const float* lse_i = lse + (g * b2 + i) * (long)b1;
  const float* del_i = delta + (g * b2 + i) * (long)b1;
  float a_kt[DV], a_y[DV], a_h = 0.f;
#pragma unroll
  for (int u = 0; u < DV; ++u) a_kt[u] = a_y[u] = 0.f;
  for (int lb = l0; lb < l1; lb += 32) {
    const int l = lb + lane;
    float Lw = 0.f, ds = 0.f;
    if (l < l1 && bias > -INFINITY) {
      const long row = (g * b1 + l) * b2 + i;
      const float s = dot_row(sk, Q + row * d, d) + bias;
      Lw = expf(s - lse_i[l]);
      ds = Lw * (dot_row(sy, dO + row * d, d) - del_i[l]);
    }
    a_h += warp_sum(ds);
    const int nl = min(32, l1 - lb);
    for (int jj = 0; jj < nl; ++jj) {
      const float lj = __shfl_sync(0xffffffffu, Lw, jj);
      const float dj = __shfl_sync(0xffffffffu, ds, jj);
      const long row = (g * b1 + lb + jj) * b2 + i;
#pragma unroll
      for (int u = 0; u < DV; ++u) {
        const int x = lane + 32 * u;
        if (x < d) {
          a_kt[u] = fmaf(dj, to_f32(Q[row * d + x]), a_kt[u]);
          a_y[u] = fmaf(lj, to_f32(dO[row * d + x]), a_y[u]);
        }
      }
    }
  }
#pragma unroll
  for (int u = 0; u < DV; ++u) {
    const int x = lane + 32 * u;
    if (x < d) {
      dkt[key * d + x] = a_kt[u] * pb.sc;
      dy[key * d + x] = a_y[u];
    }
  }
  if (lane == 0) dhs[key] = a_h;
}

// ---- R side, one warp per R row (g, k, p, q, i); one block per (g, k) ----
template <typename TIn, int DV>
__global__ void __launch_bounds__(kThreads)
    r_bwd_rows_kernel(const TIn* __restrict__ K, const TIn* __restrict__ V,
                      const float* __restrict__ qt0, const float* __restrict__ dkt,
                      const float* __restrict__ dy, const float* __restrict__ dhs,
                      float* __restrict__ rbuf, float* __restrict__ dsbuf,
                      float* __restrict__ dqt0_part, Problem pb) {
  extern __shared__ float smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int d = pb.d, b1 = pb.b1, b2 = pb.b2, c1 = pb.c1, c2 = pb.c2;
  const int k = (int)(blockIdx.x % b1);
  const long g = blockIdx.x / b1;
  float* sq = smem + warp * 3 * d;
  float* sa = sq + d;
  float* sy = sa + d;
  const TIn* Kk = K + (g * b1 + k) * (long)b2 * d;
  const TIn* Vk = V + (g * b1 + k) * (long)b2 * d;
  const int nrows = c1 * c2 * b2;
  for (int rr = warp; rr < nrows; rr += kWarps) {
    const int i = rr % b2, q = (rr / b2) % c2, p = rr / (b2 * c2);
    const long krow = (((g * b2 + i) * c1 + p) * b1 + k) * (long)c2 + q;  // Kt / dKt row
    const float* qv = qt0 + ((g * c1 + p) * b2 + i) * (long)d;
    for (int x = lane; x < d; x += 32) {
      sq[x] = qv[x] * pb.sc;
      sa[x] = dkt[krow * d + x];
      sy[x] = dy[krow * d + x];
    }
    __syncwarp();
    const float h = dhs[krow];
    const int j0 = group_start(b2, c2, q), j1 = group_start(b2, c2, q + 1);
    float* R_row = rbuf + (((g * b1 + k) * c1 + p) * b2 + i) * (long)b2;
    float* dS_row = dsbuf + (((g * b1 + k) * c1 + p) * b2 + i) * (long)b2;
    // pass 1: softmax statistics over j in q
    float m = -INFINITY, z = 0.f;
    for (int jb = j0; jb < j1; jb += 32) {
      const int j = jb + lane;
      const float s = j < j1 ? dot_row(sq, Kk + (long)j * d, d) : -INFINITY;
      const float mn = fmaxf(m, warp_max(s));
      const float alpha = (m == -INFINITY) ? 0.f : expf(m - mn);
      z = z * alpha + warp_sum(j < j1 ? expf(s - mn) : 0.f);
      m = mn;
    }
    const float lz = logf(z);
    // pass 2: R_j and dR_j (kept in dS_row), c = sum R dR
    float c = 0.f;
    for (int jb = j0; jb < j1; jb += 32) {
      const int j = jb + lane;
      float rj = 0.f, drj = 0.f;
      if (j < j1) {
        const float s = dot_row(sq, Kk + (long)j * d, d);
        const float ln_r = s - m - lz;
        rj = expf(ln_r);
        drj = dot_row(sa, Kk + (long)j * d, d) + dot_row(sy, Vk + (long)j * d, d) -
              h * (ln_r + 1.f);
        R_row[j] = rj;
        dS_row[j] = drj;
      }
      c += warp_sum(rj * drj);
    }
    __syncwarp();
    // pass 3: dS_R = R (dR - c); partial dQt0 = sc sum_j dS_R k_j
    float aq[DV];
#pragma unroll
    for (int u = 0; u < DV; ++u) aq[u] = 0.f;
    for (int jb = j0; jb < j1; jb += 32) {
      const int j = jb + lane;
      float ds = 0.f;
      if (j < j1) {
        ds = R_row[j] * (dS_row[j] - c);
        dS_row[j] = ds;
      }
      const int nj = min(32, j1 - jb);
      for (int jj = 0; jj < nj; ++jj) {
        const float dj = __shfl_sync(0xffffffffu, ds, jj);
        const TIn* kr = Kk + (long)(jb + jj) * d;
#pragma unroll
        for (int u = 0; u < DV; ++u) {
          const int x = lane + 32 * u;
          if (x < d) aq[u] = fmaf(dj, to_f32(kr[x]), aq[u]);
        }
      }
    }
    float* part = dqt0_part + ((((g * c1 + p) * b2 + i) * b1 + k) * (long)c2 + q) * d;
#pragma unroll
    for (int u = 0; u < DV; ++u) {
      const int x = lane + 32 * u;
      if (x < d) part[x] = aq[u] * pb.sc;
    }
    __syncwarp();
  }
}

// ---- R side, one warp per key token (g, k, j) ----
template <typename TIn, int DV>
__global__ void __launch_bounds__(kThreads)
    r_bwd_keys_kernel(const float* __restrict__ qt0, const float* __restrict__ dkt,
                      const float* __restrict__ dy, const float* __restrict__ rbuf,
                      const float* __restrict__ dsbuf, TIn* __restrict__ dK,
                      TIn* __restrict__ dV, Problem pb) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int d = pb.d, b1 = pb.b1, b2 = pb.b2, c1 = pb.c1, c2 = pb.c2;
  const int njb = (b2 + kWarps - 1) / kWarps;
  const int jb = (int)(blockIdx.x % njb);
  const long r = blockIdx.x / njb;
  const int k = (int)(r % b1);
  const long g = r / b1;
  const int j = jb * kWarps + warp;
  if (j >= b2) return;
  const int q = group_of(b2, c2, j);
  float ak[DV], av[DV];
#pragma unroll
  for (int u = 0; u < DV; ++u) ak[u] = av[u] = 0.f;
  for (int p = 0; p < c1; ++p) {
    for (int i = 0; i < b2; ++i) {
      const long ri = (((g * b1 + k) * c1 + p) * b2 + i) * (long)b2 + j;
      const float rj = rbuf[ri], dsj = dsbuf[ri] * pb.sc;
      const long krow = (((g * b2 + i) * c1 + p) * b1 + k) * (long)c2 + q;
      const float* qv = qt0 + ((g * c1 + p) * b2 + i) * (long)d;
#pragma unroll
      for (int u = 0; u < DV; ++u) {
        const int x = lane + 32 * u;
        if (x < d) {
          ak[u] = fmaf(rj, dkt[krow * d + x], fmaf(dsj, qv[x], ak[u]));
          av[u] = fmaf(rj, dy[krow * d + x], av[u]);
        }
      }
    }
  }
  const long row = (g * b1 + k) * b2 + j;
#pragma unroll
  for (int u = 0; u < DV; ++u) {
    const int x = lane + 32 * u;
    if (x < d) {
      dK[row * d + x] = from_f32<TIn>(ak[u]);
      dV[row * d + x] = from_f32<TIn>(av[u]);
    }
  }
}

// ---- queries, one warp per (g, p, i): dQt0 then dq of the group's rows ----
template <typename TIn, int DV>
__global__ void __launch_bounds__(kThreads)
    q_bwd_kernel(const float* __restrict__ dq1, const float* __restrict__ dqt0_part,
                 TIn* __restrict__ dQ, Problem pb) {
  // one block per (g, p, i): warp w sums the partials kq = w, w + 8, ...;
  // the eight warp sums are added in a fixed order, so the result is
  // deterministic; then the warps share the group's rows l
  __shared__ float red[kWarps][DV * 32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int d = pb.d, b1 = pb.b1, b2 = pb.b2, c1 = pb.c1, c2 = pb.c2;
  const long unit = blockIdx.x;
  const int i = (int)(unit % b2);
  const int p = (int)((unit / b2) % c1);
  const long g = unit / ((long)b2 * c1);
  float a[DV];
#pragma unroll
  for (int u = 0; u < DV; ++u) a[u] = 0.f;
  const float* part = dqt0_part + ((g * c1 + p) * b2 + i) * (long)b1 * c2 * d;
  for (int kq = warp; kq < b1 * c2; kq += kWarps) {
#pragma unroll
    for (int u = 0; u < DV; ++u) {
      const int x = lane + 32 * u;
      if (x < d) a[u] += part[(long)kq * d + x];
    }
  }
#pragma unroll
  for (int u = 0; u < DV; ++u) red[warp][lane + 32 * u] = a[u];
  __syncthreads();
#pragma unroll
  for (int u = 0; u < DV; ++u) {
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) t += red[w][lane + 32 * u];
    a[u] = t;
  }
  const int l0 = group_start(b1, c1, p), l1 = group_start(b1, c1, p + 1);
  const float inv = 1.f / (float)(l1 - l0);
  for (int l = l0 + warp; l < l1; l += kWarps) {
    const long row = (g * b1 + l) * b2 + i;
#pragma unroll
    for (int u = 0; u < DV; ++u) {
      const int x = lane + 32 * u;
      if (x < d) dQ[row * d + x] = from_f32<TIn>(dq1[row * d + x] + a[u] * inv);
    }
  }
}

inline unsigned ceil_div(long n, long m) { return (unsigned)((n + m - 1) / m); }

template <typename TIn, int DV>
cudaError_t run_bwd(const TIn* q, const TIn* k, const TIn* v, const TIn* dout, TIn* dq, TIn* dk,
                    TIn* dv, const Problem& pb, const BwdWorkspace& ws, int* status,
                    cudaStream_t stream, int* launches) {
  const int G = pb.G, b1 = pb.b1, b2 = pb.b2, c1 = pb.c1, c2 = pb.c2, d = pb.d;
  const size_t shm2 = (size_t)kWarps * 2 * d * sizeof(float);
  const size_t shm3 = (size_t)kWarps * 3 * d * sizeof(float);
  cudaError_t e = cudaSuccess;
  bool l_side_done = false, r_side_done = false;
  if constexpr (std::is_same<TIn, bf16>::value) {
    // bf16 rows of <= 128 keys: the tensor-core step one recomputes the
    // forward quantities and the tensor-core L side takes them; untiled
    // chunks of <= 128 positions take the tensor-core R side too
    if (bwd_tc_l_side_supports(pb)) {
      bf16* qt016 = reinterpret_cast<bf16*>(ws.qt016);
      bf16* kt16 = reinterpret_cast<bf16*>(ws.kt16);
      bf16* y16 = reinterpret_cast<bf16*>(ws.y16);
      const bool tc_r = bwd_tc_r_side_supports(pb);
      bf16* dkt16 = tc_r ? reinterpret_cast<bf16*>(ws.dkt16) : nullptr;
      bf16* dy16 = tc_r ? reinterpret_cast<bf16*>(ws.dy16) : nullptr;
      e = bwd_tc_recompute(q, k, v, qt016, kt16, y16, ws.hs, ws.qt0, pb, status, stream,
                           launches);
      if (e != cudaSuccess) return e;
      e = bwd_tc_l_side(q, dout, kt16, y16, ws.hs, ws.dq1, ws.dkt, ws.dy, ws.dhs, dkt16, dy16, pb,
                        status, stream, launches);
      if (e != cudaSuccess) return e;
      l_side_done = true;
      if (tc_r) {
        e = bwd_tc_r_side(qt016, k, v, dkt16, dy16, ws.dhs, ws.dqt0_part, dk, dv, pb, status,
                          stream, launches);
        if (e != cudaSuccess) return e;
        r_side_done = true;
      }
    }
  }
  if (!l_side_done) {
    // forward intermediates: Qt0, Kt, Y, Hs (fp32)
    SimtWorkspace fw{};
    fw.qt0 = ws.qt0;
    fw.kt = ws.kt;
    fw.y = ws.y;
    fw.hs = ws.hs;
    e = simt_forward<TIn, float>(q, k, v, (TIn*)nullptr, pb, fw, stream, launches, false);
    if (e != cudaSuccess) return e;
  }
  if (!l_side_done) e = timed_launch("bwd_l_rows", stream, launches, [&] {
    l_bwd_rows_kernel<TIn, DV><<<ceil_div((long)G * b2 * ceil_div(b1, kWarps), 1), kThreads,
                                 shm2, stream>>>(q, dout, ws.kt, ws.y, ws.hs, ws.dq1, ws.lse,
                                                 ws.delta, pb);
  });
  if (e != cudaSuccess) return e;
  if (!l_side_done) e = timed_launch("bwd_l_keys", stream, launches, [&] {
    l_bwd_keys_kernel<TIn, DV><<<(unsigned)((long)G * b2 * c1 * ceil_div((long)b1 * c2, kWarps)),
                                 kThreads, shm2, stream>>>(q, dout, ws.kt, ws.y, ws.hs, ws.lse,
                                                           ws.delta, ws.dkt, ws.dy, ws.dhs, pb);
  });
  if (e != cudaSuccess) return e;
  if (!r_side_done) e = timed_launch("bwd_r_rows", stream, launches, [&] {
    r_bwd_rows_kernel<TIn, DV><<<(unsigned)((long)G * b1), kThreads, shm3, stream>>>(
        k, v, ws.qt0, ws.dkt, ws.dy, ws.dhs, ws.rbuf, ws.dsbuf, ws.dqt0_part, pb);
  });
  if (e != cudaSuccess) return e;
  if (!r_side_done) e = timed_launch("bwd_r_keys", stream, launches, [&] {
    r_bwd_keys_kernel<TIn, DV><<<(unsigned)((long)G * b1 * ceil_div(b2, kWarps)), kThreads, 0,
                                 stream>>>(ws.qt0, ws.dkt, ws.dy, ws.rbuf, ws.dsbuf, dk, dv, pb);
  });
  if (e != cudaSuccess) return e;
  return timed_launch("bwd_q", stream, launches, [&] {
    q_bwd_kernel<TIn, DV><<<(unsigned)((long)G * c1 * b2), kThreads, 0, stream>>>(
        ws.dq1, ws.dqt0_part, dq, pb);
  });
}

}  // namespace

BwdWorkspaceSizes bwd_workspace_sizes(const Problem& pb) {
  BwdWorkspaceSizes s;
  const size_t G = pb.G, b1 = pb.b1, b2 = pb.b2, c1 = pb.c1, c2 = pb.c2, d = pb.d;
  const size_t N = b1 * b2;
  s.qt0 = G * c1 * b2 * d;
  s.kt = G * N * c1 * c2 * d;
  s.y = s.kt;
  s.hs = G * N * c1 * c2;
  s.lse = G * N;
  s.delta = G * N;
  s.dq1 = G * N * d;
  s.dkt = s.kt;
  s.dy = s.kt;
  s.dhs = s.hs;
  s.rbuf = G * b1 * c1 * b2 * b2;
  s.dsbuf = s.rbuf;
  s.dqt0_part = G * c1 * b2 * b1 * c2 * d;
  s.qt016 = (s.qt0 + 1) / 2;
  s.kt16 = (s.kt + 1) / 2;
  s.y16 = s.kt16;
  s.dkt16 = s.kt16;
  s.dy16 = s.kt16;
  return s;
}

template <typename TIn>
cudaError_t bwd_forward_t1(const TIn* q, const TIn* k, const TIn* v, const TIn* dout, TIn* dq,
                           TIn* dk, TIn* dv, const Problem& pb, const BwdWorkspace& ws,
                           int* status, cudaStream_t stream, int* launches) {
  if (pb.T != 1 || is_padded(pb)) return cudaErrorInvalidValue;
  if (pb.d <= 32)
    return run_bwd<TIn, 1>(q, k, v, dout, dq, dk, dv, pb, ws, status, stream, launches);
  if (pb.d <= 64)
    return run_bwd<TIn, 2>(q, k, v, dout, dq, dk, dv, pb, ws, status, stream, launches);
  if (pb.d <= 128)
    return run_bwd<TIn, 4>(q, k, v, dout, dq, dk, dv, pb, ws, status, stream, launches);
  return run_bwd<TIn, 8>(q, k, v, dout, dq, dk, dv, pb, ws, status, stream, launches);
}

template cudaError_t bwd_forward_t1<float>(const float*, const float*, const float*, const float*,
                                           float*, float*, float*, const Problem&,
                                           const BwdWorkspace&, int*, cudaStream_t, int*);
template cudaError_t bwd_forward_t1<bf16>(const bf16*, const bf16*, const bf16*, const bf16*,
                                          bf16*, bf16*, bf16*, const Problem&,
                                          const BwdWorkspace&, int*, cudaStream_t, int*);

}  // namespace monarch
