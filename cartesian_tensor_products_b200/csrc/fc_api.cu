// libflashcart: status strings, descriptor queries and the receiver row
// pointer build/validation (FlashCart App. D "Receiver-sorted forward").
#include <math.h>

#include "fc_common.cuh"

namespace fc {

int device_sm_count() {
  static DeviceFlags cache;   // the SM count per device, 0 = not yet queried
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev < 0 || dev >= kMaxDevices) return 148;
  int n = cache[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cache[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

int check_conv_desc(const fc_conv_desc* d) {
  if (!d) return FC_ERR_ARG;
  if (d->lmax_in < 0 || d->lmax_edge < 0 || d->lmax_out < 0) return FC_ERR_ARG;
  if (d->sum_paths != 0 && d->sum_paths != 1) return FC_ERR_ARG;
  if (d->channels <= 0) return FC_ERR_ARG;
  if (d->lmax_in != d->lmax_edge || d->lmax_in != d->lmax_out) return FC_ERR_UNSUPPORTED_RANK;
  if (d->lmax_in < 1 || d->lmax_in > 5) return FC_ERR_UNSUPPORTED_RANK;
  if (d->channels % 4) return FC_ERR_ALIGN;
  if (d->envelope != 0 && d->envelope != 1) return FC_ERR_ARG;
  if (d->envelope == 1 && !(d->r_cut > 0.0f && isfinite(d->r_cut) && isfinite(d->edge_scale)))
    return FC_ERR_ARG;
  return FC_OK;
}

// E = sum of the rank-0 block; gz = indicator of the rank-0 block
__global__ void readout_kernel(long long total, int NYC, int C, const float* __restrict__ z,
                               float* __restrict__ energy, float* __restrict__ gz) {
  float part = 0.0f;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const bool r0 = (i % NYC) < C;
    if (r0) part += z[i];
    if (gz) gz[i] = r0 ? 1.0f : 0.0f;
  }
  for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
  if ((threadIdx.x & 31) == 0) atomicAdd(energy, part);
}

__global__ void forces_kernel(int N, int E, const int32_t* __restrict__ recv,
                              const int32_t* __restrict__ send, const float* __restrict__ rbar,
                              float* __restrict__ F) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= E) return;
  const int u = recv[e], v = send[e];
  const float x = rbar[3 * e], y = rbar[3 * e + 1], zz = rbar[3 * e + 2];
  if (v >= 0 && v < N) {
    atomicAdd(F + 3 * v, -x); atomicAdd(F + 3 * v + 1, -y); atomicAdd(F + 3 * v + 2, -zz);
  }
  if (u >= 0 && u < N) {
    atomicAdd(F + 3 * u, x); atomicAdd(F + 3 * u + 1, y); atomicAdd(F + 3 * u + 2, zz);
  }
}

// Flags raised by the validation kernel.
enum : int { kBadRecv = 1, kUnsorted = 2, kBadSend = 4, kDegenerate = 8 };

// Thread e (0 <= e <= E) validates edge e and fills the row pointers of the
// receivers in (recv[e-1], recv[e]] with e (recv[-1] = -1, recv[E] = N),
// so each entry of a valid receiver-sorted list is written exactly once.
__global__ void build_rowptr_kernel(int N, int NS, int E, const int32_t* __restrict__ recv,
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
    if (s < 0 || s >= NS) bad |= kBadSend;
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

int fc_scalar_readout(int n_nodes, int lmax, int channels, const float* z, float* energy,
                      float* gz, fc_stream_t stream) {
  if (n_nodes < 0 || lmax < 0 || lmax > 8 || channels <= 0 || !energy) return FC_ERR_ARG;
  if (n_nodes > 0 && !z) return FC_ERR_ARG;
  if (!aligned4(energy) || (z && !aligned4(z)) || (gz && !aligned4(gz))) return FC_ERR_ALIGN;
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemsetAsync(energy, 0, sizeof(float), s) != cudaSuccess) return FC_ERR_CUDA;
  if (n_nodes == 0) return FC_OK;
  const int NYC = (lmax + 1) * (lmax + 1) * channels;
  const long long total = (long long)n_nodes * NYC;
  long long blocks = (total + 255) / 256;
  if (blocks > 4 * 148) blocks = 4 * 148;
  readout_kernel<<<(int)blocks, 256, 0, s>>>(total, NYC, channels, z, energy, gz);
  return cudaGetLastError() == cudaSuccess ? FC_OK : FC_ERR_CUDA;
}

int fc_edge_forces(int n_nodes, int n_edges, const int32_t* edge_index, const float* r_bar,
                   float* forces, fc_stream_t stream) {
  if (n_nodes < 0 || n_edges < 0 || !forces) return FC_ERR_ARG;
  if (n_edges > 0 && (!edge_index || !r_bar)) return FC_ERR_ARG;
  if (!aligned4(forces) || (r_bar && !aligned4(r_bar)) || (edge_index && !aligned4(edge_index)))
    return FC_ERR_ALIGN;
  cudaStream_t s = (cudaStream_t)stream;
  if (n_nodes > 0 && cudaMemsetAsync(forces, 0, sizeof(float) * 3 * (size_t)n_nodes, s) != cudaSuccess)
    return FC_ERR_CUDA;
  if (n_edges == 0) return FC_OK;
  forces_kernel<<<(n_edges + 255) / 256, 256, 0, s>>>(n_nodes, n_edges, edge_index,
                                                       edge_index + n_edges, r_bar, forces);
  return cudaGetLastError() == cudaSuccess ? FC_OK : FC_ERR_CUDA;
}

int fc_build_rowptr_rect(int n_nodes, int n_send, int n_edges, const int32_t* edge_index,
                         const float* edge_vec, int32_t* rowptr, int32_t* flag,
                         fc_stream_t stream) {
  if (n_nodes < 0 || n_send < 0 || n_edges < 0 || !rowptr || !flag) return FC_ERR_ARG;
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
        n_nodes, n_send, n_edges, edge_index, edge_index ? edge_index + n_edges : nullptr,
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

int fc_build_rowptr(int n_nodes, int n_edges, const int32_t* edge_index,
                    const float* edge_vec, int32_t* rowptr, int32_t* flag,
                    fc_stream_t stream) {
  return fc_build_rowptr_rect(n_nodes, n_nodes, n_edges, edge_index, edge_vec, rowptr, flag, stream);
}

}  // extern "C"
