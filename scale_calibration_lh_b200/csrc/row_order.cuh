// Ordering of a sweep CTA's 128 rows by their first unclamped candidate.
//
// Both sweep kernels evaluate a row's candidates below kfirst (the first candidate at which one
// of its 16 weights falls below the top E2M1 level) with a closed form, and the rest in full;
// a warp can take the closed form only while all of its rows can. Ordering the CTA's rows by
// kfirst groups rows that leave the clamped regime together. Any order gives the same results
// per row, but the order must be deterministic, so the sort is stable: a counting sort over
// the 127 values of kfirst (0..126), run by the CTA's first four warps (one row per thread).
//
// Usage, with every thread of the CTA passing each __syncthreads():
//   zero hist (4 x 128 ints);                               __syncthreads();
//   threads < 128: row_order_count(kf, hist);               __syncthreads();
//   warp 0: row_order_scan(hist, base);                     __syncthreads();
//   threads < 128: row_order_place(kf, hist, base, perm, kf_sorted);  __syncthreads();
// Afterwards perm[i] is the i-th row in ascending kfirst (ties in row order) and
// kf_sorted[i] its kfirst, so a warp's first row in sorted order has the warp's smallest kfirst.
#pragma once

#include <stdint.h>

namespace lhcal {

constexpr int kOrderRows = 128;

// Step 1 (threads 0..127, whole warps): rows of this warp per kfirst value.
__device__ __forceinline__ void row_order_count(int kf, int (*hist)[kOrderRows]) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t same = __match_any_sync(0xffffffffu, kf);
  if (lane == __ffs(same) - 1) hist[warp][kf] = __popc(same);
}

// Step 2 (warp 0): base[v] = rows with kfirst < v, an exclusive scan over the 128 values.
__device__ __forceinline__ void row_order_scan(const int (*hist)[kOrderRows], int* base) {
  const int lane = threadIdx.x & 31;
  int c[4], run = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int v = 4 * lane + j;
    c[j] = hist[0][v] + hist[1][v] + hist[2][v] + hist[3][v];
    run += c[j];
  }
  int incl = run;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  int b = incl - run;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    base[4 * lane + j] = b;
    b += c[j];
  }
}

// Step 3 (threads 0..127): the row's position = rows with a smaller kfirst + rows of earlier
// warps with the same one + lanes of this warp before this one with the same one.
__device__ __forceinline__ void row_order_place(int kf, const int (*hist)[kOrderRows], const int* base, int* perm,
                                                int* kf_sorted) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t same = __match_any_sync(0xffffffffu, kf);
  int pos = base[kf] + __popc(same & ((1u << lane) - 1u));
  for (int w2 = 0; w2 < warp; ++w2) pos += hist[w2][kf];
  perm[pos] = threadIdx.x;
  kf_sorted[pos] = kf;
}

}  // namespace lhcal
