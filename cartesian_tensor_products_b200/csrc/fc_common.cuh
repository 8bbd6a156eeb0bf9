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
template <int L, int G, int g>
struct VvjpGroup;
template <int L>
struct VvjpMeta;
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

// tensor-core per-rank channel mix of the ladder (fc_mix_tc.cu), C = 128.
// Operands in the tiled split layout: rows of rank l in 128-row tiles
// ts[l] .. ts[l+1] - 1, each tile 4 K chunks x (hi, lo) x 4096 floats in the
// core-matrix layout; matrices [L+1][hi, lo][16384].
struct MixTiles {
  int ts[8];   // first tile of rank l (ts[l] = total for l > L)
  int total;
};
bool mix_tc_supported(int L, int C);
MixTiles mix_tc_tiles(int L, int N);
size_t mix_tc_operand_floats(int L, int N);
size_t mix_tc_matrix_floats(int L);
// natural [N][(L+1)^2][128] -> tiled split layout (rows past each rank's end = 0)
int launch_mix_tc_split_rows(int L, int N, const float* in, float* xs, cudaStream_t s);
// mode 0: A(j, t) = M[j][t] (forward); mode 1: A(j, t) = M[t][j] (VJP)
int launch_mix_tc_split_matrix(int mode, int L, const float* M, float* ws, cudaStream_t s);
// out[n][l^2 + c][j] = sum_t A_l(j, t) x[n][l^2 + c][t] for every rank l
int launch_mix_tc(int L, int N, const float* xs, const float* ws, float* out, cudaStream_t s);
// natural -> transposed split tiles (channels x rows, K-major along rows)
int launch_mix_tc_split_cols(int L, int N, const float* in, float* xs, cudaStream_t s);
// Mbar[l][k][j] += sum over the rows of rank l of a[row][k] b[row][j] (both transposed split)
int launch_wgrad_tc(int L, int N, const float* as, const float* bs, float* Mbar, cudaStream_t s);

}  // namespace fc
