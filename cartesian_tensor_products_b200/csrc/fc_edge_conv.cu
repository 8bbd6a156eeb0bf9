// libflashcart: receiver-sorted edge convolution, forward (FlashCart
// Sec. 4 Eq. (1), Algorithm 1): C ABI entry point and the rank 1-4
// instantiations; the kernel templates and their design notes are in
// fc_edge_conv.cuh, rank 5 is instantiated in fc_edge_conv_L5.cu.
#include "fc_edge_conv.cuh"
#include "generated/fc_fwd_L1.cuh"
#include "generated/fc_fwd_L2.cuh"
#include "generated/fc_fwd_L3.cuh"
#include "generated/fc_fwd_L4.cuh"

namespace fc {
int launch_fwd_rank5(const ConvArgs& a, cudaStream_t s);
}  // namespace fc

using namespace fc;

extern "C" int fc_edge_conv_rect(const fc_conv_desc* d, int n_nodes, int n_send, int n_edges,
                                 const int32_t* rowptr, const int32_t* edge_index,
                                 const float* edge_vec, const float* x, const float* w, float* z,
                                 fc_stream_t stream) {
  int st = check_conv_desc(d);
  if (st != FC_OK) return st;
  if (n_nodes < 0 || n_send < 0 || n_edges < 0) return FC_ERR_ARG;
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
  a.n_send = n_send;
  a.n_edges = n_edges;
  a.C = C;
  a.ntiles = (C + 127) / 128;
  a.xrow = (L + 1) * (L + 1);
  a.zrow = out_row(L, d->sum_paths);
  a.P = num_paths(L);
  a.sum_paths = d->sum_paths;
  a.envelope = d->envelope;
  a.r_cut = d->r_cut;
  a.edge_scale = d->edge_scale;
  if ((long long)n_nodes * a.ntiles > 0x7fffffffLL) return FC_ERR_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  if (d->sum_paths) {
    if (cudaMemsetAsync(z, 0, sizeof(float) * (size_t)n_nodes * a.zrow * C, s) != cudaSuccess)
      return FC_ERR_CUDA;
  }
  switch (L) {
    case 1: return launch_fwd<1>(a, s);
    case 2: return launch_fwd<2>(a, s);
    case 3: return launch_fwd<3>(a, s);
    case 4: return launch_fwd<4>(a, s);
    case 5: return launch_fwd_rank5(a, s);
    default: return FC_ERR_UNSUPPORTED_RANK;
  }
}

extern "C" int fc_edge_conv(const fc_conv_desc* d, int n_nodes, int n_edges,
                            const int32_t* rowptr, const int32_t* edge_index,
                            const float* edge_vec, const float* x, const float* w, float* z,
                            fc_stream_t stream) {
  return fc_edge_conv_rect(d, n_nodes, n_nodes, n_edges, rowptr, edge_index, edge_vec, x, w, z,
                           stream);
}

extern "C" size_t fc_edge_conv_workspace_size(const fc_conv_desc* d, int n_nodes, int n_edges) {
  (void)d;
  (void)n_nodes;
  (void)n_edges;
  return 0;   // the receiver sums stay on chip; no call of the convolution family needs scratch
}
