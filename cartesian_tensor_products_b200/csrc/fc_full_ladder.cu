// libflashcart: the full correlation ladder, forward.
//
// FlashCart (arXiv 2610.06409) Sec. 5 Eq. (2): the products keep every
// coupling path and a learned map mixes paths and channels per output rank,
//   phi_1[l,c,:] = W1_l A[l,c,:]
//   B_q[eta,c,k] = f_eta(phi_{q-1}[l1,:,k], A[l2,:,k])_c              (q = 2..order)
//   phi_q[l,c,j] = sum_{eta -> l} sum_k Wq_l[j][eta_l C + k] B_q[eta,c,k]
//   z = phi_1 + ... + phi_order.
// B_q is written in the convolution's output layout ([N][sum_l (2l+1) P_l][C],
// slot zoff(l) + c P_l + eta), so the P_l C inputs of one (node, component)
// row of the mix are one contiguous run: each mix is a GEMM per rank with
// K = P_l C (K = C for phi_1), register-tiled FP32 (64 rows x 128 channels
// per CTA, 4 x 8 outputs per thread) with z += phi_q in its epilogue.  The
// products are channel-diagonal: one thread per channel, generated
// straight-line code per path (exact coefficients).
//
// At C = 128 the maps run on the tcgen05 tensor cores (fc_mix_tc.cu,
// three-term TF32 split): the product kernel writes B_q straight into the
// FP32 tile layout the map kernel stages (input k of a rank-l row = eta_l C +
// channel), phi_1 reads A copied into the same tiles; z is summed
// from the states at the end.  Rows past the last node of a tile are never
// written: the MMA column of such a row depends on that row alone and is not
// stored.
#include "fc_common.cuh"
#include "fc_device.cuh"
#include "fc_tc.cuh"
#include "generated/fc_ladder_L1.cuh"
#include "generated/fc_ladder_L2.cuh"
#include "generated/fc_ladder_L3.cuh"
#include "generated/fc_ladder_L4.cuh"

namespace fc {

namespace {

constexpr int kFullChunk = 4;   // nodes per thread in the product kernel

template <int L>
__global__ void __launch_bounds__(128) full_tp_paths_kernel(int N, int C, const float* __restrict__ phi,
                                                            const float* __restrict__ A,
                                                            float* __restrict__ Bz) {
  using TP = LadderTP<L>;
  const int k = blockIdx.y * blockDim.x + threadIdx.x;
  if (k >= C) return;
  const int n0 = blockIdx.x * kFullChunk;
  const int n1 = min(N, n0 + kFullChunk);
  for (int n = n0; n < n1; ++n) {
    const size_t base = (size_t)n * TP::NY * C + k;
    float a[TP::NY], b[TP::NY];
#pragma unroll
    for (int i = 0; i < TP::NY; ++i) {
      a[i] = __ldg(phi + base + (size_t)i * C);
      b[i] = __ldg(A + base + (size_t)i * C);
    }
    TP::fwd_paths(a, b, Bz + (size_t)n * TP::ZROW * C + k, C);
  }
}

// The same products at C = 128, written as the FP32 path-mix operand
// (component-major PathGeom tiles, k_l = 4 P_l).
// A warp takes 8 consecutive nodes x 4 consecutive channels: for one output
// (path, component) its 32 values are exactly one 128-byte core matrix
// (8 rows x 4 inputs), so every store instruction writes one full line.
template <int L>
__global__ void __launch_bounds__(256, 2) full_tp_tiled_kernel(PathGeom g, const float* __restrict__ phi,
                                                            const float* __restrict__ A,
                                                            float* __restrict__ xs) {
  using TP = LadderTP<L>;
  constexpr int C = 128;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int n = 8 * blockIdx.x + (lane >> 2);
  const int k = 32 * blockIdx.y + 4 * warp + (lane & 3);
  if (n >= g.N) return;
  const int kq = k >> 5, kk = k & 31;   // chunk within a path, input within the chunk
  const int r = n & 127, nblk = n >> 7;
  const size_t base = (size_t)n * TP::NY * C + k;
  float a[TP::NY], b[TP::NY];
#pragma unroll
  for (int i = 0; i < TP::NY; ++i) {
    a[i] = __ldg(phi + base + (size_t)i * C);
    b[i] = __ldg(A + base + (size_t)i * C);
  }
  const int cofs = tc::core_offset(r, kk, 128);
  TP::fwd_paths_to(a, b, [&](int l3, int c, int eta, float v) {
    const int kc = pg_kc(g, l3);
    xs[pg_xbase(g, l3) + (long long)(c * g.nb + nblk) * kc * 4096 + (eta * 4 + kq) * 4096 + cofs] = v;
  });
}

// z = sum of the order states
__global__ void __launch_bounds__(256) full_sum_kernel(size_t plane4, int order,
                                                       const float4* __restrict__ states,
                                                       float4* __restrict__ z) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < plane4;
       i += (size_t)gridDim.x * blockDim.x) {
    float4 acc = __ldg(states + i);
    for (int q = 1; q < order; ++q) {
      const float4 v = __ldg(states + (size_t)q * plane4 + i);
      acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
    }
    z[i] = acc;
  }
}

// Rows of rank l: i in [0, N(2l+1)), node n = i / (2l+1), component c.  The
// input row of (n, c) starts at (n in_row + off[l] + c cmul[l]) C and holds
// K[l] values; the rank's map is W + woff[l], [C][K[l]] row-major.
struct FullMixGeom {
  int N, C, NY, in_row, L;
  int off[6], cmul[6], K[6], woff[6];
};

constexpr int kFBM = 64, kFBN = 128, kFBK = 32;

__global__ void __launch_bounds__(256) full_mix_kernel(const FullMixGeom g, const float* __restrict__ in,
                                                       const float* __restrict__ W,
                                                       float* __restrict__ out, float* __restrict__ z) {
  __shared__ __align__(16) float As[kFBK][kFBM + 4];
  __shared__ __align__(16) float Bs[kFBK][kFBN + 4];
  const int l = blockIdx.z;
  if (l > g.L) return;
  const int w = 2 * l + 1;
  const int R = g.N * w;
  const int r0 = blockIdx.x * kFBM;
  if (r0 >= R) return;
  const int C = g.C, K = g.K[l], off = g.off[l], cmul = g.cmul[l];
  const float* Wl = W + g.woff[l];
  const int j0 = blockIdx.y * kFBN;
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;   // 16 x 16 threads: 8 channels x 4 rows each
  float acc[4][8];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.0f;
  for (int t0 = 0; t0 < K; t0 += kFBK) {
#pragma unroll
    for (int s = 0; s < 2; ++s) {   // A: 64 rows x 32 t, stored t-major
      const int idx = tid + s * 256;
      const int rr = idx >> 3, tq = (idx & 7) * 4;
      const int i = r0 + rr;
      float4 v = zero4();
      if (i < R && t0 + tq < K) {
        const int n = i / w, c = i - (i / w) * w;
        v = __ldg(reinterpret_cast<const float4*>(in + ((size_t)n * g.in_row + off + c * cmul) * C + t0 + tq));
      }
      As[tq + 0][rr] = v.x; As[tq + 1][rr] = v.y; As[tq + 2][rr] = v.z; As[tq + 3][rr] = v.w;
    }
#pragma unroll
    for (int s = 0; s < 4; ++s) {   // B: 32 t x 128 j from W[j][t]
      const int idx = tid + s * 256;
      const int jj = idx >> 3, tq = (idx & 7) * 4;
      float4 v = zero4();
      if (j0 + jj < C && t0 + tq < K)
        v = __ldg(reinterpret_cast<const float4*>(Wl + (size_t)(j0 + jj) * K + t0 + tq));
      Bs[tq + 0][jj] = v.x; Bs[tq + 1][jj] = v.y; Bs[tq + 2][jj] = v.z; Bs[tq + 3][jj] = v.w;
    }
    __syncthreads();
#pragma unroll 8
    for (int t = 0; t < kFBK; ++t) {
      const float4 a = *reinterpret_cast<const float4*>(&As[t][ty * 4]);
      const float4 b0 = *reinterpret_cast<const float4*>(&Bs[t][tx * 8]);
      const float4 b1 = *reinterpret_cast<const float4*>(&Bs[t][tx * 8 + 4]);
      const float av[4] = {a.x, a.y, a.z, a.w};
      const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = r0 + ty * 4 + i;
    if (r >= R) continue;
    const int n = r / w, c = r - (r / w) * w;
    const size_t base = ((size_t)n * g.NY + l * l + c) * C;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int j = j0 + tx * 8 + h * 4;
      if (j >= C) continue;
      const float4 v = make_float4(acc[i][h * 4], acc[i][h * 4 + 1], acc[i][h * 4 + 2], acc[i][h * 4 + 3]);
      *reinterpret_cast<float4*>(out + base + j) = v;
      float4 zz = *reinterpret_cast<float4*>(z + base + j);
      zz.x += v.x; zz.y += v.y; zz.z += v.z; zz.w += v.w;
      *reinterpret_cast<float4*>(z + base + j) = zz;
    }
  }
}

int launch_full_mix(const FullMixGeom& g, const float* in, const float* W, float* out, float* z,
                    cudaStream_t s) {
  const int Rmax = g.N * (2 * g.L + 1);
  dim3 grid((Rmax + kFBM - 1) / kFBM, (g.C + kFBN - 1) / kFBN, g.L + 1);
  full_mix_kernel<<<grid, 256, 0, s>>>(g, in, W, out, z);
  return cudaGetLastError() == cudaSuccess ? FC_OK : FC_ERR_CUDA;
}

template <int L>
int launch_tp_paths(int N, int C, const float* phi, const float* A, float* Bz, cudaStream_t s) {
  dim3 grid((N + kFullChunk - 1) / kFullChunk, (C + 127) / 128);
  full_tp_paths_kernel<L><<<grid, 128, 0, s>>>(N, C, phi, A, Bz);
  return cudaGetLastError() == cudaSuccess ? FC_OK : FC_ERR_CUDA;
}

int tp_paths_dispatch(int L, int N, int C, const float* phi, const float* A, float* Bz, cudaStream_t s) {
  switch (L) {
    case 1: return launch_tp_paths<1>(N, C, phi, A, Bz, s);
    case 2: return launch_tp_paths<2>(N, C, phi, A, Bz, s);
    case 3: return launch_tp_paths<3>(N, C, phi, A, Bz, s);
    case 4: return launch_tp_paths<4>(N, C, phi, A, Bz, s);
  }
  return FC_ERR_UNSUPPORTED_RANK;
}

int tp_tiled_dispatch(int L, const PathGeom& g, const float* phi, const float* A, float* xs,
                      cudaStream_t s) {
  const dim3 grid((g.N + 7) / 8, 4);
  switch (L) {
    case 1: full_tp_tiled_kernel<1><<<grid, 256, 0, s>>>(g, phi, A, xs); break;
    case 2: full_tp_tiled_kernel<2><<<grid, 256, 0, s>>>(g, phi, A, xs); break;
    case 3: full_tp_tiled_kernel<3><<<grid, 256, 0, s>>>(g, phi, A, xs); break;
    case 4: full_tp_tiled_kernel<4><<<grid, 256, 0, s>>>(g, phi, A, xs); break;
    default: return FC_ERR_UNSUPPORTED_RANK;
  }
  return cudaGetLastError() == cudaSuccess ? FC_OK : FC_ERR_CUDA;
}

// paths into each output rank (all l1, l2 <= L)
void rank_paths(int L, int* Pl) {
  for (int l3 = 0; l3 <= L; ++l3) {
    Pl[l3] = 0;
    for (int l1 = 0; l1 <= L; ++l1)
      for (int l2 = 0; l2 <= L; ++l2)
        if (l3 >= (l1 > l2 ? l1 - l2 : l2 - l1) && l3 <= l1 + l2 && ((l1 + l2 + l3) & 1) == 0) ++Pl[l3];
  }
}

// tile geometries of the tensor-core path: phi_1 (K = C per rank) and the
// path-separated steps (K = P_l C)
void tc_geoms(int L, int N, PathGeom& g1, PathGeom& gq) {
  int Pl[6] = {0, 0, 0, 0, 0, 0}, k1[5] = {0, 0, 0, 0, 0}, kq[5] = {0, 0, 0, 0, 0};
  rank_paths(L, Pl);
  for (int l = 0; l <= L; ++l) {
    k1[l] = 4;
    kq[l] = 4 * Pl[l];
  }
  g1 = path_geom(L, N, k1);
  gq = path_geom(L, N, kq);
}

size_t tc_operand_floats(const PathGeom& gq) { return (size_t)pg_xbase(gq, gq.L + 1); }

int check_full_desc(const fc_ladder_desc* d) {
  if (!d) return FC_ERR_ARG;
  if (d->channels <= 0 || d->order < 1 || d->lmax < 0) return FC_ERR_ARG;
  if (d->lmax < 1 || d->lmax > 4) return FC_ERR_UNSUPPORTED_RANK;
  if (d->channels % 4) return FC_ERR_ALIGN;
  return FC_OK;
}

}  // namespace
}  // namespace fc

using namespace fc;

extern "C" size_t fc_full_ladder_workspace_size(const fc_ladder_desc* d, int n_nodes) {
  if (check_full_desc(d) != FC_OK || n_nodes < 0) return 0;
  if (mix_tc_supported(d->lmax, d->channels)) {
    PathGeom g1, gq;
    tc_geoms(d->lmax, n_nodes, g1, gq);
    return sizeof(float) * (tc_operand_floats(gq) + (size_t)pg_wbase(gq, gq.L + 1));
  }
  if (d->order < 2) return 0;
  return sizeof(float) * (size_t)n_nodes * out_row(d->lmax, 0) * d->channels;
}

extern "C" int fc_full_ladder(const fc_ladder_desc* d, int n_nodes, const float* A, const float* W1,
                              const float* Wq, float* states, float* z, void* workspace,
                              size_t ws_bytes, fc_stream_t stream) {
  int st = check_full_desc(d);
  if (st != FC_OK) return st;
  if (n_nodes < 0) return FC_ERR_ARG;
  if (n_nodes == 0) return FC_OK;
  const int L = d->lmax, C = d->channels, order = d->order;
  if (!A || !W1 || !states || !z || (order > 1 && !Wq)) return FC_ERR_ARG;
  if (!aligned16(A) || !aligned16(W1) || !aligned16(states) || !aligned16(z) ||
      (order > 1 && !aligned16(Wq)))
    return FC_ERR_ALIGN;
  const size_t need = fc_full_ladder_workspace_size(d, n_nodes);
  if (need > 0 && (!workspace || ws_bytes < need)) return FC_ERR_WORKSPACE;
  if (need > 0 && !aligned16(workspace)) return FC_ERR_ALIGN;
  cudaStream_t s = (cudaStream_t)stream;
  if (mix_tc_supported(L, C)) {
    // tensor-core maps, then z = phi_1 + ... + phi_order
    PathGeom g1, gq;
    tc_geoms(L, n_nodes, g1, gq);
    float* xs = static_cast<float*>(workspace);
    float* wsm = xs + tc_operand_floats(gq);
    const size_t plane = (size_t)n_nodes * (L + 1) * (L + 1) * C;
    const size_t wq_step = (size_t)C * num_paths(L) * C;
    if ((st = launch_path_split_rows(g1, A, xs, s)) != FC_OK ||
        (st = launch_path_split_map(g1, W1, wsm, s)) != FC_OK ||
        (st = launch_path_mix_tc(g1, xs, wsm, states, s)) != FC_OK)
      return st;
    for (int q = 2; q <= order; ++q) {
      if ((st = tp_tiled_dispatch(L, gq, states + (size_t)(q - 2) * plane, A, xs, s)) != FC_OK ||
          (st = launch_path_split_map(gq, Wq + (size_t)(q - 2) * wq_step, wsm, s)) != FC_OK ||
          (st = launch_path_mix_tc(gq, xs, wsm, states + (size_t)(q - 1) * plane, s)) != FC_OK)
        return st;
    }
    full_sum_kernel<<<8 * device_sm_count(), 256, 0, s>>>(plane / 4, order,
                                                         reinterpret_cast<const float4*>(states),
                                                         reinterpret_cast<float4*>(z));
    return cudaGetLastError() == cudaSuccess ? FC_OK : FC_ERR_CUDA;
  }
  const int NY = (L + 1) * (L + 1);
  const size_t plane = (size_t)n_nodes * NY * C;
  int Pl[6] = {0, 0, 0, 0, 0, 0};
  rank_paths(L, Pl);
  const int P = num_paths(L);
  if (cudaMemsetAsync(z, 0, sizeof(float) * plane, s) != cudaSuccess) return FC_ERR_CUDA;
  // phi_1 = W1_l A per rank (natural rows, K = C)
  FullMixGeom g1{};
  g1.N = n_nodes; g1.C = C; g1.NY = NY; g1.in_row = NY; g1.L = L;
  for (int l = 0; l <= L; ++l) {
    g1.off[l] = l * l; g1.cmul[l] = 1; g1.K[l] = C; g1.woff[l] = l * C * C;
  }
  if ((st = launch_full_mix(g1, A, W1, states, z, s)) != FC_OK) return st;
  // later steps: path-separated products, then the path+channel map of each rank
  FullMixGeom gq{};
  gq.N = n_nodes; gq.C = C; gq.NY = NY; gq.in_row = out_row(L, 0); gq.L = L;
  int zoff = 0, roff = 0;
  for (int l = 0; l <= L; ++l) {
    gq.off[l] = zoff; gq.cmul[l] = Pl[l]; gq.K[l] = Pl[l] * C; gq.woff[l] = roff * C * C;
    zoff += (2 * l + 1) * Pl[l];
    roff += Pl[l];
  }
  float* Bz = static_cast<float*>(workspace);
  for (int q = 2; q <= order; ++q) {
    if ((st = tp_paths_dispatch(L, n_nodes, C, states + (size_t)(q - 2) * plane, A, Bz, s)) != FC_OK ||
        (st = launch_full_mix(gq, Bz, Wq + (size_t)(q - 2) * C * P * C, states + (size_t)(q - 1) * plane,
                              z, s)) != FC_OK)
      return st;
  }
  return FC_OK;
}
