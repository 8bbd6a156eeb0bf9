// libflashcart: receiver-sorted edge convolution, forward.
//
// FlashCart (arXiv 2610.06409) Sec. 4 Eq. (1) and Algorithm 1:
//   z_{u eta k} = sum_{e: u_e = u} w_{e eta k} f_eta(x_{v_e k}, y_e),
//   y_e = T(r-hat_e) shared by all channels.
// Every receiver's sums are accumulated on chip and stored once.
//
// B200 design.  A CTA holds G warps; warp g owns a fixed group of output
// rows (path, component), chosen offline so that every warp does the same
// number of FMAs, and covers 128 channels of one receiver (4 per lane, so
// every global access is a coalesced 16-byte vector).  The CTA walks a
// strided list of (receiver, 128-channel tile) units.  For each chunk of up
// to 32 incoming edges a warp first forms, lane-per-edge, the entries of
// M_eta[a][b] = sum_b2 K_eta[a][b][b2] y_e,b2 its rows need and parks them
// in a warp-private shared-memory row; then it walks the edges, loading the
// sender's feature rows (L2-resident) and the edge's path weights
// (streamed from HBM, one edge ahead in registers) and accumulating
// w * (M x) with every M entry read as a shared-memory broadcast.
#include "fc_common.cuh"
#include "fc_device.cuh"
#include "generated/fc_fwd_L2.cuh"
#include "generated/fc_fwd_L3.cuh"
#include "generated/fc_fwd_L4.cuh"

namespace fc {

struct ConvArgs {
  const int32_t* rowptr;
  const int32_t* send;
  const float* vec;
  const float* x;
  const float* w;
  float* z;
  int n_nodes, n_edges, C, ntiles, xrow, zrow, P, sum_paths;
};

template <class Grp>
__device__ __forceinline__ void load_edge(const ConvArgs& a, int v, int e, int k0, bool act,
                                          float4 (&xr)[Grp::NX], float4 (&wr)[Grp::NWP]) {
  if (act && v >= 0) {
    Grp::load_x(a.x + (size_t)v * a.xrow * a.C + k0, a.C, xr);
    Grp::load_w(a.w + (size_t)e * a.P * a.C + k0, a.C, wr);
  } else {
#pragma unroll
    for (int i = 0; i < Grp::NX; ++i) xr[i] = zero4();
#pragma unroll
    for (int i = 0; i < Grp::NWP; ++i) wr[i] = zero4();
  }
}

template <class Grp>
__device__ __forceinline__ void fwd_warp(const ConvArgs& a, float* __restrict__ mbuf,
                                         int* __restrict__ sbuf, int lane) {
  const int n_units = a.n_nodes * a.ntiles;
  for (int unit = blockIdx.x; unit < n_units; unit += gridDim.x) {
    const int u = unit / a.ntiles;
    const int tile = unit - u * a.ntiles;
    const int k0 = tile * 128 + lane * 4;
    const bool act = k0 < a.C;
    int e0 = a.rowptr[u], e1 = a.rowptr[u + 1];
    e0 = e0 < 0 ? 0 : (e0 > a.n_edges ? a.n_edges : e0);
    e1 = e1 < e0 ? e0 : (e1 > a.n_edges ? a.n_edges : e1);
    float4 acc[Grp::NA];
#pragma unroll
    for (int i = 0; i < Grp::NA; ++i) acc[i] = zero4();

    for (int cs = e0; cs < e1; cs += 32) {
      const int n = (e1 - cs) < 32 ? (e1 - cs) : 32;
      if (lane < n) {
        const int e = cs + lane;
        const float rx = a.vec[3 * e], ry = a.vec[3 * e + 1], rz = a.vec[3 * e + 2];
        const float inv = 1.0f / sqrtf(rx * rx + ry * ry + rz * rz);
        Grp::make_m(rx * inv, ry * inv, rz * inv, mbuf + lane * Grp::MSTRIDE);
        const int v = a.send[e];
        sbuf[lane] = (v >= 0 && v < a.n_nodes) ? v : -1;
      }
      __syncwarp();
      // ping-pong between two register buffers, one edge of look-ahead
      float4 xa[Grp::NX], wa[Grp::NWP], xb[Grp::NX], wb[Grp::NWP];
      load_edge<Grp>(a, sbuf[0], cs, k0, act, xa, wa);
      for (int j = 0; j < n; j += 2) {
        if (j + 1 < n) load_edge<Grp>(a, sbuf[j + 1], cs + j + 1, k0, act, xb, wb);
        Grp::accum(acc, xa, wa, mbuf + j * Grp::MSTRIDE);
        if (j + 1 >= n) break;
        if (j + 2 < n) load_edge<Grp>(a, sbuf[j + 2], cs + j + 2, k0, act, xa, wa);
        Grp::accum(acc, xb, wb, mbuf + (j + 1) * Grp::MSTRIDE);
      }
      __syncwarp();
    }
    if (act) Grp::store(a.z + (size_t)u * a.zrow * a.C + k0, a.C, a.sum_paths, acc);
  }
}

template <int L, int g>
__device__ __forceinline__ void dispatch_fwd(int warp, const ConvArgs& a, float* mbuf,
                                             int* sbuf, int lane) {
  if constexpr (g < FwdMeta<L>::G) {
    if (warp == g) {
      fwd_warp<FwdGroup<L, FwdMeta<L>::G, g>>(a, mbuf, sbuf, lane);
      return;
    }
    dispatch_fwd<L, g + 1>(warp, a, mbuf, sbuf, lane);
  }
}

template <int L>
__global__ void __launch_bounds__(FwdMeta<L>::G * 32, 1)
    edge_conv_fwd_kernel(const ConvArgs a) {
  extern __shared__ __align__(16) float smem[];
  constexpr int MS = FwdMeta<L>::MAXSTRIDE;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* mbuf = smem + warp * 32 * MS;
  int* sbuf = reinterpret_cast<int*>(smem + FwdMeta<L>::G * 32 * MS) + warp * 32;
  dispatch_fwd<L, 0>(warp, a, mbuf, sbuf, lane);
}

template <int L>
static size_t fwd_smem_bytes() {
  return sizeof(float) * (size_t)FwdMeta<L>::G * 32 * FwdMeta<L>::MAXSTRIDE +
         sizeof(int) * (size_t)FwdMeta<L>::G * 32;
}

template <int L>
static int launch_fwd(const ConvArgs& a, cudaStream_t s) {
  const size_t smem = fwd_smem_bytes<L>();
  static int configured[64] = {0};
  static int blocks_per_sm[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return FC_ERR_CUDA;
  if (!configured[dev]) {
    if (cudaFuncSetAttribute(edge_conv_fwd_kernel<L>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
      return FC_ERR_CUDA;
    int nb = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, edge_conv_fwd_kernel<L>,
                                                      FwdMeta<L>::G * 32, smem) != cudaSuccess)
      return FC_ERR_CUDA;
    blocks_per_sm[dev] = nb > 0 ? nb : 1;
    configured[dev] = 1;
  }
  const long long units = (long long)a.n_nodes * a.ntiles;
  long long grid = (long long)device_sm_count() * blocks_per_sm[dev];
  if (grid > units) grid = units;
  if (grid < 1) grid = 1;
  edge_conv_fwd_kernel<L><<<(int)grid, FwdMeta<L>::G * 32, smem, s>>>(a);
  return cudaGetLastError() == cudaSuccess ? FC_OK : FC_ERR_CUDA;
}

}  // namespace fc

using namespace fc;

extern "C" int fc_edge_conv(const fc_conv_desc* d, int n_nodes, int n_edges,
                            const int32_t* rowptr, const int32_t* edge_index,
                            const float* edge_vec, const float* x, const float* w, float* z,
                            fc_stream_t stream) {
  int st = check_conv_desc(d);
  if (st != FC_OK) return st;
  if (n_nodes < 0 || n_edges < 0) return FC_ERR_ARG;
  if (n_nodes == 0) return n_edges == 0 ? FC_OK : FC_ERR_ARG;
  if (!rowptr || !x || !z) return FC_ERR_ARG;
  if (n_edges > 0 && (!edge_index || !edge_vec || !w)) return FC_ERR_ARG;
  if (!aligned16(x) || !aligned16(z) || (w && !aligned16(w)) || !aligned4(rowptr) ||
      (edge_index && !aligned4(edge_index)) || (edge_vec && !aligned4(edge_vec)))
    return FC_ERR_ALIGN;
  const int L = d->lmax_in;
  const int C = d->channels;
  ConvArgs a;
  a.rowptr = rowptr;
  a.send = edge_index ? edge_index + n_edges : nullptr;
  a.vec = edge_vec;
  a.x = x;
  a.w = w;
  a.z = z;
  a.n_nodes = n_nodes;
  a.n_edges = n_edges;
  a.C = C;
  a.ntiles = (C + 127) / 128;
  a.xrow = (L + 1) * (L + 1);
  a.zrow = out_row(L, d->sum_paths);
  a.P = num_paths(L);
  a.sum_paths = d->sum_paths;
  if ((long long)n_nodes * a.ntiles > 0x7fffffffLL) return FC_ERR_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  if (d->sum_paths) {
    if (cudaMemsetAsync(z, 0, sizeof(float) * (size_t)n_nodes * a.zrow * C, s) != cudaSuccess)
      return FC_ERR_CUDA;
  }
  switch (L) {
    case 2: return launch_fwd<2>(a, s);
    case 3: return launch_fwd<3>(a, s);
    case 4: return launch_fwd<4>(a, s);
    default: return FC_ERR_UNSUPPORTED_RANK;
  }
}
