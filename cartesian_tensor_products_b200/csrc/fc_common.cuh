// Host-side helpers shared by the libflashcart translation units.
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "flashcart.h"

namespace fc {

template <int L, int G, int g>
struct FwdGroup;
template <int L>
struct FwdMeta;
template <int L>
struct Direction;
template <int L, int G, int g>
struct VjpGroup;
template <int L>
struct VjpMeta;
template <int L>
struct LadderTP;

inline bool aligned16(const void* p) {
  return (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}
inline bool aligned4(const void* p) {
  return (reinterpret_cast<uintptr_t>(p) & 3u) == 0;
}

// number of paths / output row length for lmax_in = lmax_edge = lmax_out = L
inline int num_paths(int L) {
  int n = 0;
  for (int l3 = 0; l3 <= L; ++l3)
    for (int l1 = 0; l1 <= L; ++l1)
      for (int l2 = 0; l2 <= L; ++l2)
        if (l3 >= (l1 > l2 ? l1 - l2 : l2 - l1) && l3 <= l1 + l2 &&
            ((l1 + l2 + l3) & 1) == 0)
          ++n;
  return n;
}

inline int out_row(int L, int sum_paths) {
  if (sum_paths) return (L + 1) * (L + 1);
  int n = 0;
  for (int l3 = 0; l3 <= L; ++l3)
    for (int l1 = 0; l1 <= L; ++l1)
      for (int l2 = 0; l2 <= L; ++l2)
        if (l3 >= (l1 > l2 ? l1 - l2 : l2 - l1) && l3 <= l1 + l2 &&
            ((l1 + l2 + l3) & 1) == 0)
          n += 2 * l3 + 1;
  return n;
}

// SM count and occupancy are cached per device
int device_sm_count();

// validates the parts of a convolution descriptor this build supports
int check_conv_desc(const fc_conv_desc* d);

// tensor-core per-rank channel mix of the ladder (fc_mix_tc.cu), C = 128:
// mode 0: out = in M^T per rank; mode 1: out = in M per rank
bool mix_tc_supported(int L, int C);
int launch_mix_tc(int mode, int L, int N, const float* in, const float* M, float* out,
                  cudaStream_t s);

}  // namespace fc
