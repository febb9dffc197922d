// Row permutation between raster and Monarch token order.
#include "layout.cuh"

#include <cstdint>

#include "timing.cuh"

namespace monarch {
namespace {

// One thread per unit of a row; consecutive threads cover consecutive units
// of one row, so each row moves as one contiguous read and one contiguous
// write.  UNITS > 0 fixes the units per row at compile time (a shift).
// Up to three tensors per launch (blockIdx.y picks the pair).
struct RowPairs {
  const void* src[3];
  void* dst[3];
};

constexpr int kPermDepth = 4;

// I: the index type, int when every unit index fits (a 32-bit division per
// unit instead of a 64-bit one), else long.
template <typename U, int UNITS, typename I>
__global__ void __launch_bounds__(256)
    permute_rows_kernel(RowPairs pairs, const int* __restrict__ table, I total, int N,
                        int units_rt, bool to_monarch) {
  const int units = UNITS > 0 ? UNITS : units_rt;
  const U* __restrict__ src = static_cast<const U*>(pairs.src[blockIdx.y]);
  U* __restrict__ dst = static_cast<U*>(pairs.dst[blockIdx.y]);
  // kPermDepth units per thread and pass, every load issued before the stores
  const I stride = (I)gridDim.x * blockDim.x;
  for (I base = (I)blockIdx.x * blockDim.x + threadIdx.x; base < total;
       base += stride * kPermDepth) {
    I from[kPermDepth], to[kPermDepth];
    U val[kPermDepth];
#pragma unroll
    for (int r = 0; r < kPermDepth; ++r) {
      const I idx = base + r * stride;
      if (idx < total) {
        const I row = idx / units;
        const int c = (int)(idx - row * units);
        const I g = row / N;
        const int m = (int)(row - g * N);
        const I n = __ldg(table + m);
        const I mi = (g * N + m) * units + c, ni = (g * N + n) * units + c;
        from[r] = to_monarch ? ni : mi;
        to[r] = to_monarch ? mi : ni;
        val[r] = src[from[r]];
      }
    }
#pragma unroll
    for (int r = 0; r < kPermDepth; ++r)
      if (base + r * stride < total) dst[to[r]] = val[r];
  }
}

template <typename U, int UNITS>
cudaError_t launch(const RowPairs& pairs, int npairs, const int* table, long G, int N,
                   int row_bytes, bool to_monarch, cudaStream_t stream, int* launches) {
  const int units = row_bytes / (int)sizeof(U);
  const long total = G * N * (long)units;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long want = (total + 256L * kPermDepth - 1) / (256L * kPermDepth);
  const int grid = (int)(want < 16L * sms ? want : 16L * sms);
  return timed_launch("permute_rows", stream, launches, [&] {
    if (total < (1L << 31) - 256L * grid * kPermDepth)  // no index overflows int
      permute_rows_kernel<U, UNITS, int><<<dim3(grid, npairs), 256, 0, stream>>>(
          pairs, table, (int)total, N, units, to_monarch);
    else
      permute_rows_kernel<U, UNITS, long><<<dim3(grid, npairs), 256, 0, stream>>>(
          pairs, table, total, N, units, to_monarch);
  });
}

// Padding copies: one thread per unit of a destination row.
template <typename U>
__global__ void __launch_bounds__(256)
    pad_rows_kernel(RowPairs pairs, long total, int rows_dst, int N, int n_src, int real_lo,
                    int units, bool to_grid) {
  const U* __restrict__ src = static_cast<const U*>(pairs.src[blockIdx.y]);
  U* __restrict__ dst = static_cast<U*>(pairs.dst[blockIdx.y]);
  for (long idx = (long)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (long)gridDim.x * blockDim.x) {
    const long row = idx / units;
    const int c = (int)(idx - row * units);
    const long g = row / rows_dst;
    const int r = (int)(row - g * rows_dst);
    if (to_grid) {  // r is a grid row
      const int rs = r - real_lo;
      U val;
      if (rs >= 0 && rs < n_src) {
        val = src[(g * n_src + rs) * units + c];
      } else {
        memset(&val, 0, sizeof(U));
      }
      dst[idx] = val;
    } else {  // r is a real row
      dst[idx] = src[(g * N + r + real_lo) * units + c];
    }
  }
}

template <typename U>
cudaError_t launch_pad(const RowPairs& pairs, int npairs, long G, int N, int n_src, int real_lo,
                       int row_bytes, bool to_grid, cudaStream_t stream, int* launches) {
  const int units = row_bytes / (int)sizeof(U);
  const int rows_dst = to_grid ? N : n_src;
  const long total = G * rows_dst * (long)units;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long want = (total + 255) / 256;
  const int grid = (int)(want < 16L * sms ? want : 16L * sms);
  return timed_launch("pad_rows", stream, launches, [&] {
    pad_rows_kernel<U><<<dim3(grid, npairs), 256, 0, stream>>>(pairs, total, rows_dst, N, n_src,
                                                               real_lo, units, to_grid);
  });
}

}  // namespace

void video_perm_table(const VideoPerm& vp, int* table) {
  int m = 0;
  for (int x0 = 0; x0 < vp.s[0]; ++x0)
    for (int x1 = 0; x1 < vp.s[1]; ++x1)
      for (int x2 = 0; x2 < vp.s[2]; ++x2)
        table[m++] = (int)(x0 * vp.t[0] + x1 * vp.t[1] + x2 * vp.t[2]);
}

cudaError_t permute_rows(const void* const* src, void* const* dst, int n, const int* table,
                         long G, int N, int row_bytes, bool to_monarch, cudaStream_t stream,
                         int* launches) {
  if (n < 1 || n > 3 || G < 1 || N < 1 || row_bytes < 1) return cudaErrorInvalidValue;
  RowPairs pairs = {};
  uintptr_t a = static_cast<uintptr_t>(row_bytes);
  for (int i = 0; i < n; ++i) {
    pairs.src[i] = src[i];
    pairs.dst[i] = dst[i];
    a |= reinterpret_cast<uintptr_t>(src[i]) | reinterpret_cast<uintptr_t>(dst[i]);
  }
#define MONARCH_PERMUTE(U, UNITS) \
  return launch<U, UNITS>(pairs, n, table, G, N, row_bytes, to_monarch, stream, launches)
  if (a % 16 == 0) {
    switch (row_bytes / 16) {  // d = 64 / 128 in bf16 or fp32
      case 8: MONARCH_PERMUTE(uint4, 8);
      case 16: MONARCH_PERMUTE(uint4, 16);
      case 32: MONARCH_PERMUTE(uint4, 32);
      default: MONARCH_PERMUTE(uint4, 0);
    }
  }
  if (a % 8 == 0) MONARCH_PERMUTE(uint2, 0);
  if (a % 4 == 0) MONARCH_PERMUTE(uint32_t, 0);
  if (a % 2 == 0) MONARCH_PERMUTE(uint16_t, 0);
  MONARCH_PERMUTE(uint8_t, 0);
#undef MONARCH_PERMUTE
}

cudaError_t pad_rows(const void* const* src, void* const* dst, int n, long G, int N, int n_src,
                     int real_lo, int row_bytes, bool to_grid, cudaStream_t stream,
                     int* launches) {
  if (n < 1 || n > 3 || G < 1 || N < 1 || n_src < 1 || real_lo < 0 || real_lo + n_src > N ||
      row_bytes < 1)
    return cudaErrorInvalidValue;
  RowPairs pairs = {};
  uintptr_t a = static_cast<uintptr_t>(row_bytes);
  for (int i = 0; i < n; ++i) {
    pairs.src[i] = src[i];
    pairs.dst[i] = dst[i];
    a |= reinterpret_cast<uintptr_t>(src[i]) | reinterpret_cast<uintptr_t>(dst[i]);
  }
#define MONARCH_PAD(U) \
  return launch_pad<U>(pairs, n, G, N, n_src, real_lo, row_bytes, to_grid, stream, launches)
  if (a % 16 == 0) MONARCH_PAD(uint4);
  if (a % 8 == 0) MONARCH_PAD(uint2);
  if (a % 4 == 0) MONARCH_PAD(uint32_t);
  if (a % 2 == 0) MONARCH_PAD(uint16_t);
  MONARCH_PAD(uint8_t);
#undef MONARCH_PAD
}

}  // namespace monarch
