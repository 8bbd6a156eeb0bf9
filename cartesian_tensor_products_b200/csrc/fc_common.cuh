// Host-side helpers shared by the libflashcart translation units.
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <atomic>

#include "flashcart.h"

namespace fc {

// Host-side per-device set-up flags (kernel attributes, cached queries).
// Concurrent first calls from several host threads may each run the set-up
// (the CUDA runtime calls involved are thread-safe and idempotent); the flag
// itself is an atomic, so there is no data race.
constexpr int kMaxDevices = 64;
using DeviceFlags = std::atomic<int>[kMaxDevices];

// Raises a kernel's dynamic shared-memory limit to `bytes` once per device.
template <class Kernel>
inline int set_smem_once(DeviceFlags& done, Kernel kernel, size_t bytes) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FC_ERR_CUDA;
  if (done[dev].load(std::memory_order_acquire)) return FC_OK;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) !=
      cudaSuccess)
    return FC_ERR_CUDA;
  done[dev].store(1, std::memory_order_release);
  return FC_OK;
}

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

// Odd-J (Levi-Civita) paths: l1, l2 >= 1, |l1 - l2| <= l3 <= l1 + l2 - 1,
// l1 + l2 + l3 odd.  Their kernels are instantiated under rank key L + kOddKey.
constexpr int kOddKey = 16;

inline bool odd_admissible(int l1, int l2, int l3) {
  return l1 >= 1 && l2 >= 1 && l3 >= (l1 > l2 ? l1 - l2 : l2 - l1) && l3 <= l1 + l2 - 1 &&
         ((l1 + l2 + l3) & 1) == 1;
}

inline int num_odd_paths(int L) {
  int n = 0;
  for (int l3 = 0; l3 <= L; ++l3)
    for (int l1 = 0; l1 <= L; ++l1)
      for (int l2 = 0; l2 <= L; ++l2) n += odd_admissible(l1, l2, l3);
  return n;
}

inline int odd_out_row(int L, int sum_paths) {
  if (sum_paths) return (L + 1) * (L + 1);
  int n = 0;
  for (int l3 = 0; l3 <= L; ++l3)
    for (int l1 = 0; l1 <= L; ++l1)
      for (int l2 = 0; l2 <= L; ++l2)
        if (odd_admissible(l1, l2, l3)) n += 2 * l3 + 1;
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

// Tensor-core path + channel map of the full ladder (fc_mix_tc.cu), C = 128.
// Rows of rank l (node n, component c) carry K = 32 k_l inputs (k_l = 4 P_l:
// P_l paths x 128 channels).  They form 128-row tiles t_l .. t_{l+1} - 1,
// component-major: tile t_l + c nb + n / 128 holds component c of nodes
// 128 (n / 128) + 0..127 (nb = ceil(N / 128); rows past node N - 1 unused).
// A tile is k_l FP32 blocks of 4096 floats (128 rows x 32 inputs,
// core-matrix layout), and rank l's tiles start at float pg_xbase(l) of the
// operand buffer.  The map of rank l ([128][K]) is split into TF32: k_l hi
// then k_l lo blocks of the same layout from float pg_wbase(l).
//
// A rank may carry several maps (e_l > 1: one per path into rank l, the
// full-ladder VJP's B_bar = p_bar Wq_l, path by path): each (map, tile) pair
// is a unit of work, the maps of rank l one after the other, and map e of
// rank l writes row (node n, component c) at row n orow + ooff(l) + c e_l + e
// of the output (orow = NY and e_l = 1: the node layout; e_l = P_l and orow =
// the convolution's output row: one slot per path).
struct PathGeom {
  int N, NY, L, nb;
  int t1, t2, t3, t4, t5;   // first tile of ranks 1..5 (t_{L+1} = all tiles)
  int k0, k1, k2, k3, k4;   // K chunks per row of ranks 0..4
  int e0, e1, e2, e3, e4;   // maps of ranks 0..4
  int orow;                 // output row length (in 128-channel rows)
};
__host__ __device__ __forceinline__ int pg_ts(const PathGeom& g, int l) {
  return l <= 0 ? 0 : l == 1 ? g.t1 : l == 2 ? g.t2 : l == 3 ? g.t3 : l == 4 ? g.t4 : g.t5;
}
__host__ __device__ __forceinline__ int pg_kc(const PathGeom& g, int l) {
  return l == 0 ? g.k0 : l == 1 ? g.k1 : l == 2 ? g.k2 : l == 3 ? g.k3 : g.k4;
}
__host__ __device__ __forceinline__ int pg_rank(const PathGeom& g, int t) {
  return (g.L >= 1 && t >= g.t1) + (g.L >= 2 && t >= g.t2) + (g.L >= 3 && t >= g.t3) +
         (g.L >= 4 && t >= g.t4);
}
__host__ __device__ __forceinline__ long long pg_xbase(const PathGeom& g, int l) {
  long long b = 0;
#pragma unroll
  for (int r = 0; r < 5; ++r)
    if (r < l) b += (long long)(pg_ts(g, r + 1) - pg_ts(g, r)) * pg_kc(g, r) * 4096;
  return b;
}
__host__ __device__ __forceinline__ int pg_pe(const PathGeom& g, int l) {
  return l == 0 ? g.e0 : l == 1 ? g.e1 : l == 2 ? g.e2 : l == 3 ? g.e3 : g.e4;
}
// maps of rank l start at float pg_wbase(l) (each map: k_l hi then k_l lo blocks)
__host__ __device__ __forceinline__ long long pg_wbase(const PathGeom& g, int l) {
  long long b = 0;
#pragma unroll
  for (int r = 0; r < 5; ++r)
    if (r < l) b += (long long)pg_kc(g, r) * pg_pe(g, r) * 8192;
  return b;
}
// first output row of rank l within a node's row
__host__ __device__ __forceinline__ int pg_ooff(const PathGeom& g, int l) {
  int o = 0;
#pragma unroll
  for (int r = 0; r < 5; ++r)
    if (r < l) o += (2 * r + 1) * pg_pe(g, r);
  return o;
}
// kc[l] = K chunks per row of rank l (l <= L <= 4); one map per rank, node-layout output
PathGeom path_geom(int L, int N, const int* kc);
// the same with pe[l] maps of rank l and path-slot output rows
PathGeom path_geom_maps(int L, int N, const int* kc, const int* pe);
// natural [N][(L+1)^2][32 k] -> FP32 operand tiles with k_l = k = 4 or 8 for every rank
int launch_path_split_rows(const PathGeom& g, const float* in, float* xs, cudaStream_t s);
// the maps, rank l's ([128 e_l][32 k_l] row-major, map e = rows 128 e ..) at
// W + 4096 sum_{l'<l} k_l' e_l', -> split blocks at ws + pg_wbase(l)
int launch_path_split_map(const PathGeom& g, const float* W, float* ws, cudaStream_t s);
// e_l maps per rank: map e of rank l is the transposed block e of
// Wq_l = [32 k_l][128 e_l] (rank l at Wq + 4096 sum_{l'<l} k_l' e_l'):
// A(j', t) = Wq_l[t][e 128 + j'] (k_l = 4 or 8)
int launch_path_split_map_t(const PathGeom& g, const float* Wq, float* ws, cudaStream_t s);
// out[n][l^2 + c][j] = sum_k W_l[j][k] x_l[(n, c)][k]
int launch_path_mix_tc(const PathGeom& g, const float* xs, const float* ws, float* out, cudaStream_t s);

// Weight gradient of a per-rank map from FP32 rows on tcgen05 (fc_mix_tc.cu):
//   Wb_l[j][e 128 + k] += sum_{rows i = (n, c) of rank l} a[i][j] b_e[i][k]
// C = 128.  Row (n, c) of a is at float (n sa + l^2 + c) 128 (node layout);
// row (n, c) of b_e at (n sb + ob_l + c pe_l + e) 128 (e < pe_l: the node
// layout with pe = 1, or the path slots of the convolution's output layout);
// Wb_l is [128][pe_l 128] row-major at Wb + wo_l.  Adds atomically.
struct WgGeom {
  int N, L, sa, sb;
  int ob0, ob1, ob2, ob3, ob4;
  int pe0, pe1, pe2, pe3, pe4;
  int wo0, wo1, wo2, wo3, wo4;
};
__host__ __device__ __forceinline__ int wg_ob(const WgGeom& g, int l) {
  return l == 0 ? g.ob0 : l == 1 ? g.ob1 : l == 2 ? g.ob2 : l == 3 ? g.ob3 : g.ob4;
}
__host__ __device__ __forceinline__ int wg_pe(const WgGeom& g, int l) {
  return l == 0 ? g.pe0 : l == 1 ? g.pe1 : l == 2 ? g.pe2 : l == 3 ? g.pe3 : g.pe4;
}
__host__ __device__ __forceinline__ int wg_wo(const WgGeom& g, int l) {
  return l == 0 ? g.wo0 : l == 1 ? g.wo1 : l == 2 ? g.wo2 : l == 3 ? g.wo3 : g.wo4;
}
int launch_rows_wgrad_tc(const WgGeom& g, const float* a, const float* b, float* Wb, cudaStream_t s);
// both operands in the node layout, one [128][128] block per rank at l 128^2
inline WgGeom node_wg_geom(int L, int N) {
  const int NY = (L + 1) * (L + 1);
  WgGeom g{N, L, NY, NY, 0, 1, 4, 9, 16, 1, 1, 1, 1, 1, 0, 16384, 2 * 16384, 3 * 16384, 4 * 16384};
  return g;
}

}  // namespace fc
