// libflashcart: status strings, descriptor queries and the receiver row
// pointer build/validation (FlashCart App. D "Receiver-sorted forward").
#include <math.h>

#include "fc_common.cuh"

namespace fc {

int device_sm_count() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev < 0 || dev >= 64) return 148;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

int check_conv_desc(const fc_conv_desc* d) {
  if (!d) return FC_ERR_ARG;
  if (d->lmax_in < 0 || d->lmax_edge < 0 || d->lmax_out < 0) return FC_ERR_ARG;
  if (d->sum_paths != 0 && d->sum_paths != 1) return FC_ERR_ARG;
  if (d->channels <= 0) return FC_ERR_ARG;
  if (d->lmax_in != d->lmax_edge || d->lmax_in != d->lmax_out) return FC_ERR_UNSUPPORTED_RANK;
  if (d->lmax_in < 2 || d->lmax_in > 4) return FC_ERR_UNSUPPORTED_RANK;
  if (d->channels % 4) return FC_ERR_ALIGN;
  return FC_OK;
}

// Flags raised by the validation kernel.
enum : int { kBadRecv = 1, kUnsorted = 2, kBadSend = 4, kDegenerate = 8 };

// Thread e (0 <= e <= E) validates edge e and fills the row pointers of the
// receivers in (recv[e-1], recv[e]] with e (recv[-1] = -1, recv[E] = N),
// so each entry of a valid receiver-sorted list is written exactly once.
__global__ void build_rowptr_kernel(int N, int E, const int32_t* __restrict__ recv,
                                    const int32_t* __restrict__ send,
                                    const float* __restrict__ vec,
                                    int32_t* __restrict__ rowptr, int32_t* __restrict__ flag) {
  const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (e > E) return;
  int bad = 0;
  int cur = N, prev = -1;
  if (e < E) {
    cur = recv[e];
    if (cur < 0 || cur >= N) { bad |= kBadRecv; cur = cur < 0 ? 0 : N - 1; }
    const int s = send[e];
    if (s < 0 || s >= N) bad |= kBadSend;
    if (vec) {
      const float x = vec[3 * e], y = vec[3 * e + 1], z = vec[3 * e + 2];
      const float r2 = x * x + y * y + z * z;
      if (!(r2 > 0.0f) || !isfinite(r2)) bad |= kDegenerate;
    }
  }
  if (e > 0) {
    prev = recv[e - 1];
    prev = prev < 0 ? 0 : (prev >= N ? N - 1 : prev);
    if (e < E && recv[e - 1] > recv[e]) bad |= kUnsorted;
  }
  for (int u = prev + 1; u <= cur && u <= N; ++u)
    if (u >= 0) rowptr[u] = (int32_t)e;
  if (bad) atomicOr(flag, bad);
}

}  // namespace fc

using namespace fc;

extern "C" {

const char* fc_status_string(int status) {
  switch (status) {
    case FC_OK: return "ok";
    case FC_ERR_ARG: return "invalid argument";
    case FC_ERR_CSR: return "edge list is not a valid receiver-sorted graph";
    case FC_ERR_DEGENERATE_EDGE: return "edge vector of zero or non-finite length";
    case FC_ERR_UNSUPPORTED_RANK: return "rank combination not supported by this build";
    case FC_ERR_ALIGN: return "pointer not 16-byte aligned or channels not a multiple of 4";
    case FC_ERR_CUDA: return "CUDA runtime error";
    case FC_ERR_WORKSPACE: return "workspace missing or too small";
    default: return "unknown status";
  }
}

int fc_version(void) { return 100; }

int fc_conv_num_paths(const fc_conv_desc* d) {
  if (check_conv_desc(d) != FC_OK) return -1;
  return num_paths(d->lmax_in);
}

int fc_conv_out_row(const fc_conv_desc* d) {
  if (check_conv_desc(d) != FC_OK) return -1;
  return out_row(d->lmax_out, d->sum_paths);
}

int fc_conv_path(const fc_conv_desc* d, int p, int* l1, int* l2, int* l3) {
  if (check_conv_desc(d) != FC_OK || !l1 || !l2 || !l3) return FC_ERR_ARG;
  const int L = d->lmax_in;
  int n = 0;
  for (int c = 0; c <= L; ++c)
    for (int a = 0; a <= L; ++a)
      for (int b = 0; b <= L; ++b)
        if (c >= (a > b ? a - b : b - a) && c <= a + b && ((a + b + c) & 1) == 0) {
          if (n == p) { *l1 = a; *l2 = b; *l3 = c; return FC_OK; }
          ++n;
        }
  return FC_ERR_ARG;
}

int fc_build_rowptr(int n_nodes, int n_edges, const int32_t* edge_index,
                    const float* edge_vec, int32_t* rowptr, int32_t* flag,
                    fc_stream_t stream) {
  if (n_nodes < 0 || n_edges < 0 || !rowptr || !flag) return FC_ERR_ARG;
  if (n_edges > 0 && !edge_index) return FC_ERR_ARG;
  if (!aligned4(rowptr) || !aligned4(flag) || (edge_index && !aligned4(edge_index)) ||
      (edge_vec && !aligned4(edge_vec)))
    return FC_ERR_ALIGN;
  if (n_nodes == 0 && n_edges > 0) return FC_ERR_CSR;
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemsetAsync(flag, 0, sizeof(int32_t), s) != cudaSuccess) return FC_ERR_CUDA;
  if (n_nodes == 0) {
    if (cudaMemsetAsync(rowptr, 0, sizeof(int32_t), s) != cudaSuccess) return FC_ERR_CUDA;
  } else {
    const long long threads = (long long)n_edges + 1;
    const int block = 256;
    const int grid = (int)((threads + block - 1) / block);
    build_rowptr_kernel<<<grid, block, 0, s>>>(
        n_nodes, n_edges, edge_index, edge_index ? edge_index + n_edges : nullptr,
        edge_vec, rowptr, flag);
    if (cudaGetLastError() != cudaSuccess) return FC_ERR_CUDA;
  }
  int32_t h = 0;
  if (cudaMemcpyAsync(&h, flag, sizeof(int32_t), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return FC_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return FC_ERR_CUDA;
  if (h & (kBadRecv | kUnsorted | kBadSend)) return FC_ERR_CSR;
  if (h & kDegenerate) return FC_ERR_DEGENERATE_EDGE;
  return FC_OK;
}

}  // extern "C"
