// Token reordering between a video latent's raster order and the Monarch
// order of an aligned block layout (MonarchRT summary, "Key claims" and
// "Method": blocks aligned with the (f, h, w) axes).
#pragma once

#include <cuda_runtime.h>

namespace monarch {

// A layout as three axes in Monarch order: Monarch token
// m = (x0 * s1 + x1) * s2 + x2 is raster token x0*t0 + x1*t1 + x2*t2, where
// s are the axis sizes and t their raster strides in tokens.
struct VideoPerm {
  int s[3];
  long t[3];
};

// Raster index of every Monarch token (N = s0*s1*s2 entries).
void video_perm_table(const VideoPerm& vp, int* table);

// For each of the n (1-3) tensor pairs, in one launch: copies whole rows
// (row_bytes each) of G blocks of N rows from src[i] to dst[i]: dst row m =
// src row table[m] when to_monarch, else dst row table[m] = src row m.
// table is a device array of N raster indices (a permutation of 0..N-1);
// sources and destinations must not overlap.  Rows move in the widest unit
// (16, 8, 4, 2 or 1 bytes) that divides row_bytes and every base address.
cudaError_t permute_rows(const void* const* src, void* const* dst, int n, const int* table,
                         long G, int N, int row_bytes, bool to_monarch, cudaStream_t stream,
                         int* launches);

// Padding: for each of the n (1-3) tensor pairs, in one launch.  to_grid:
// dst holds G blocks of N rows and src G blocks of n_src rows; dst row m of
// a block = src row m - real_lo of the same block when that is in
// [0, n_src), zeros otherwise.  !to_grid: the reverse, dst (n_src rows per
// block) row r = src (N rows per block) row r + real_lo.  Rows move in the
// widest unit that divides row_bytes and every base address.
cudaError_t pad_rows(const void* const* src, void* const* dst, int n, long G, int N, int n_src,
                     int real_lo, int row_bytes, bool to_grid, cudaStream_t stream,
                     int* launches);

}  // namespace monarch
