// libflashcart: VJP of the full correlation ladder.
//
// FlashCart (arXiv 2610.06409) Sec. 5 Eq. (2), the full ladder of
// fc_full_ladder (every coupling path kept, a learned per-rank map mixing
// paths and channels), differentiated by reverse accumulation through its
// steps.  Every phi_q feeds z, so the running gradient pbar of phi_q starts
// at gz; going down from q = order:
//   Wq_bar_l[j][eta C + k] += sum_rows pbar[row][j] B_q[row][eta C + k]    (rows of rank l)
//   Bbar_q[row][eta C + k]  = sum_j pbar[row][j] Wq_l[j][eta C + k]
//   pbar_{q-1} = gz + the product VJP of B_q = f(phi_{q-1}, A) applied to Bbar_q,
//   A_bar     += the product VJP's A side
// (App. C Eq. C1 per path, with B_q recomputed from the saved phi_{q-1});
// then the first map: W1_bar_l += pbar_1^T A, A_bar += pbar_1 W1_l.
//
// Layouts.  B_q and Bbar_q use the convolution's output layout
// ([N][sum_l (2l+1) P_l][C], slot zoff(l) + c P_l + eta), where the P_l C
// inputs of one (node, component) row of rank l form one contiguous run, so
// every map is a GEMM over the rows of a rank: the register-tiled FP32
// kernels below (128 x 128 per CTA, 8 x 8 outputs per thread), except that at
// C = 128 the transposed map B_bar = p_bar Wq_l runs on the tcgen05 tensor
// cores (fc_mix_tc.cu's path map with one map per path).
// The weight gradients reduce over the rows (1024-row chunks per CTA, one
// atomic add per entry per chunk; not bitwise reproducible).  The products
// are channel-diagonal: one thread per channel walks a chunk of nodes with
// generated straight-line code (exact coefficients).
#include "fc_common.cuh"
#include "fc_device.cuh"
#include "generated/fc_ladder_L1.cuh"
#include "generated/fc_ladder_L2.cuh"
#include "generated/fc_ladder_L3.cuh"
#include "generated/fc_ladder_L4.cuh"

namespace fc {

namespace {

// Rows of rank l are i in [0, N(2l+1)): node n = i / (2l+1), component c;
// the row starts at float (n stride + off[l] + c cmul[l]) C of its array and
// holds wid[l] values (a multiple of 4).
struct RowLayout {
  int stride;
  int off[5], cmul[5], wid[5];
};

__device__ __forceinline__ size_t row_at(const RowLayout& g, int i, int l, int C) {
  const int w = 2 * l + 1;
  const int n = i / w;
  const int c = i - n * w;
  return ((size_t)n * g.stride + g.off[l] + (size_t)c * g.cmul[l]) * C;
}

constexpr int kVBM = 128, kVBN = 128, kVBK = 16;   // CTA tile of the row GEMMs
constexpr int kVRows = 1024;         // rows per CTA of the weight-gradient GEMMs (split K)
constexpr int kVChunk = 8;           // nodes per thread of the product VJP

// Shared inner product of the row GEMMs: a 128 x 128 tile, 256 threads, each
// thread 8 x 8 outputs (rows ty*4 + {0..3} and 64 + ty*4 + {0..3}, columns
// likewise from tx), the column pairs in packed FP32x2 accumulators.  As is
// k-major ([k][m]) and Bs is [k][n], so every thread reads two float4 of each
// per k (broadcast within a row of the warp, consecutive across it).
struct VTile {
  float As[2][kVBK][kVBM];
  float Bs[2][kVBK][kVBN];
};

__device__ __forceinline__ void vtile_mma(const VTile& sm, int buf, int tx, int ty, float2 (&acc)[8][4]) {
#pragma unroll
  for (int k = 0; k < kVBK; ++k) {
    const float4 a0 = *reinterpret_cast<const float4*>(&sm.As[buf][k][ty * 4]);
    const float4 a1 = *reinterpret_cast<const float4*>(&sm.As[buf][k][64 + ty * 4]);
    const float4 b0 = *reinterpret_cast<const float4*>(&sm.Bs[buf][k][tx * 4]);
    const float4 b1 = *reinterpret_cast<const float4*>(&sm.Bs[buf][k][64 + tx * 4]);
    const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
    const float2 bv[4] = {make_float2(b0.x, b0.y), make_float2(b0.z, b0.w), make_float2(b1.x, b1.y),
                          make_float2(b1.z, b1.w)};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float2 aa = make_float2(av[i], av[i]);
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = __ffma2_rn(aa, bv[j], acc[i][j]);
    }
  }
}

// row index of accumulator i and column index of accumulator pair j
__device__ __forceinline__ int vrow(int ty, int i) { return (i < 4 ? 0 : 64) + ty * 4 + (i & 3); }
__device__ __forceinline__ int vcol(int tx, int j) { return (j < 2 ? 0 : 64) + tx * 4 + 2 * (j & 1); }

// out_l[row][m] (+)= sum_{t < C} in[row][t] Bm_l[t][m]
// in: layout `ai` (width C), out: layout `ao` (width ao.wid[l]),
// Bm_l: [C][ao.wid[l]] row-major at Bm + boff[l].
template <bool ACC>
__global__ void __launch_bounds__(256, 2) rows_gemm_kernel(int N, int C, int L, RowLayout ai, RowLayout ao,
                                                           const float* __restrict__ in,
                                                           const float* __restrict__ Bm, long long boff0,
                                                           long long boff1, long long boff2,
                                                           long long boff3, long long boff4,
                                                           float* __restrict__ out) {
  __shared__ __align__(16) VTile sm;
  const int l = blockIdx.z;
  if (l > L) return;
  const int R = N * (2 * l + 1);
  const int r0 = blockIdx.x * kVBM;
  const int W = ao.wid[l];
  const int m0 = blockIdx.y * kVBN;
  if (r0 >= R || m0 >= W) return;
  const long long boff = l == 0 ? boff0 : l == 1 ? boff1 : l == 2 ? boff2 : l == 3 ? boff3 : boff4;
  const float* Bl = Bm + boff;
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  // global -> register prefetch of one K step: two float4 of each operand
  const int ar0 = tid >> 2, aq = tid & 3;                 // A: rows ar0, ar0 + 64; k quad aq
  const int bk = tid >> 5, bq = tid & 31;                 // B: k rows bk, bk + 8; n quad bq
  const float* arow0 = r0 + ar0 < R ? in + row_at(ai, r0 + ar0, l, C) : nullptr;
  const float* arow1 = r0 + ar0 + 64 < R ? in + row_at(ai, r0 + ar0 + 64, l, C) : nullptr;
  float4 pa0, pa1, pb0, pb1;
  auto fetch = [&](int t0) {
    const int ka = t0 + 4 * aq;
    pa0 = (arow0 && ka < C) ? __ldg(reinterpret_cast<const float4*>(arow0 + ka)) : zero4();
    pa1 = (arow1 && ka < C) ? __ldg(reinterpret_cast<const float4*>(arow1 + ka)) : zero4();
    const int n = m0 + 4 * bq;
    pb0 = (t0 + bk < C && n < W) ? __ldg(reinterpret_cast<const float4*>(Bl + (size_t)(t0 + bk) * W + n)) : zero4();
    pb1 = (t0 + bk + 8 < C && n < W) ? __ldg(reinterpret_cast<const float4*>(Bl + (size_t)(t0 + bk + 8) * W + n))
                                     : zero4();
  };
  auto stash = [&](int buf) {
    sm.As[buf][4 * aq + 0][ar0] = pa0.x; sm.As[buf][4 * aq + 1][ar0] = pa0.y;
    sm.As[buf][4 * aq + 2][ar0] = pa0.z; sm.As[buf][4 * aq + 3][ar0] = pa0.w;
    sm.As[buf][4 * aq + 0][ar0 + 64] = pa1.x; sm.As[buf][4 * aq + 1][ar0 + 64] = pa1.y;
    sm.As[buf][4 * aq + 2][ar0 + 64] = pa1.z; sm.As[buf][4 * aq + 3][ar0 + 64] = pa1.w;
    *reinterpret_cast<float4*>(&sm.Bs[buf][bk][4 * bq]) = pb0;
    *reinterpret_cast<float4*>(&sm.Bs[buf][bk + 8][4 * bq]) = pb1;
  };
  float2 acc[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = make_float2(0.0f, 0.0f);
  fetch(0);
  stash(0);
  __syncthreads();
  int buf = 0;
  for (int t0 = 0; t0 < C; t0 += kVBK) {
    const bool more = t0 + kVBK < C;
    if (more) fetch(t0 + kVBK);
    vtile_mma(sm, buf, tx, ty, acc);
    if (more) stash(buf ^ 1);
    __syncthreads();
    buf ^= 1;
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = r0 + vrow(ty, i);
    if (r >= R) continue;
    float* o = out + row_at(ao, r, l, C);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int m = m0 + vcol(tx, 2 * h);
      if (m >= W) continue;
      float4 v = make_float4(acc[i][2 * h].x, acc[i][2 * h].y, acc[i][2 * h + 1].x, acc[i][2 * h + 1].y);
      if (ACC) {
        const float4 p = *reinterpret_cast<const float4*>(o + m);
        v.x += p.x; v.y += p.y; v.z += p.z; v.w += p.w;
      }
      *reinterpret_cast<float4*>(o + m) = v;
    }
  }
}

// Wb_l[j][m] += sum_{rows of rank l} a[row][j] b[row][m]
// a: layout `la` (width C), b: layout `lb` (width lb.wid[l]),
// Wb_l: [C][lb.wid[l]] row-major at Wb + woff[l].  Each CTA reduces kVRows
// rows (split K) and adds its tile with one atomic per entry.
__global__ void __launch_bounds__(256, 2) rows_wgrad_kernel(int N, int C, int L, RowLayout la, RowLayout lb,
                                                            const float* __restrict__ a,
                                                            const float* __restrict__ b, float* __restrict__ Wb,
                                                            long long woff0, long long woff1, long long woff2,
                                                            long long woff3, long long woff4) {
  __shared__ __align__(16) VTile sm;
  const int l = blockIdx.z;
  if (l > L) return;
  const int R = N * (2 * l + 1);
  const int i0 = blockIdx.x * kVRows;
  if (i0 >= R) return;
  const int i1 = min(R, i0 + kVRows);
  const int W = lb.wid[l];
  const int jt = (C + kVBM - 1) / kVBM;
  const int j0 = (blockIdx.y % jt) * kVBM;
  const int m0 = (blockIdx.y / jt) * kVBN;
  if (m0 >= W) return;
  const long long woff = l == 0 ? woff0 : l == 1 ? woff1 : l == 2 ? woff2 : l == 3 ? woff3 : woff4;
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int kr = tid >> 5, q = tid & 31;   // rows kr, kr + 8 of the K step; column quad q
  float4 pa0, pa1, pb0, pb1;
  auto fetch = [&](int t0) {
    const int ra = t0 + kr, rb = t0 + kr + 8;
    const int j = j0 + 4 * q, m = m0 + 4 * q;
    pa0 = (ra < i1 && j < C) ? __ldg(reinterpret_cast<const float4*>(a + row_at(la, ra, l, C) + j)) : zero4();
    pa1 = (rb < i1 && j < C) ? __ldg(reinterpret_cast<const float4*>(a + row_at(la, rb, l, C) + j)) : zero4();
    pb0 = (ra < i1 && m < W) ? __ldg(reinterpret_cast<const float4*>(b + row_at(lb, ra, l, C) + m)) : zero4();
    pb1 = (rb < i1 && m < W) ? __ldg(reinterpret_cast<const float4*>(b + row_at(lb, rb, l, C) + m)) : zero4();
  };
  auto stash = [&](int buf) {
    *reinterpret_cast<float4*>(&sm.As[buf][kr][4 * q]) = pa0;
    *reinterpret_cast<float4*>(&sm.As[buf][kr + 8][4 * q]) = pa1;
    *reinterpret_cast<float4*>(&sm.Bs[buf][kr][4 * q]) = pb0;
    *reinterpret_cast<float4*>(&sm.Bs[buf][kr + 8][4 * q]) = pb1;
  };
  float2 acc[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = make_float2(0.0f, 0.0f);
  fetch(i0);
  stash(0);
  __syncthreads();
  int buf = 0;
  for (int t0 = i0; t0 < i1; t0 += kVBK) {
    const bool more = t0 + kVBK < i1;
    if (more) fetch(t0 + kVBK);
    vtile_mma(sm, buf, tx, ty, acc);
    if (more) stash(buf ^ 1);
    __syncthreads();
    buf ^= 1;
  }
  float* Wl = Wb + woff;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int j = j0 + vrow(ty, i);
    if (j >= C) continue;
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const int m = m0 + vcol(tx, h);
      if (m < W) {
        atomicAdd(Wl + (size_t)j * W + m, acc[i][h].x);
        atomicAdd(Wl + (size_t)j * W + m + 1, acc[i][h].y);
      }
    }
  }
}

// Product VJP of one step, channel-diagonal, every path with its own output
// gradient (Bbar in the convolution's output layout):
//   pbn[n,:,k]  = gz[n,:,k] + d<Bbar, f(phi, A)>/dphi
//   Abar[n,:,k] +=            d<Bbar, f(phi, A)>/dA
template <int L>
__global__ void __launch_bounds__(128) full_tp_vjp_kernel(int N, int C, const float* __restrict__ phi,
                                                          const float* __restrict__ A,
                                                          const float* __restrict__ Bbar,
                                                          const float* __restrict__ gz,
                                                          float* __restrict__ pbn, float* __restrict__ Abar) {
  using TP = LadderTP<L>;
  const int k = blockIdx.y * blockDim.x + threadIdx.x;
  if (k >= C) return;
  int zoff[L + 1], Pl[L + 1];
  {
    int o = 0;
#pragma unroll
    for (int l3 = 0; l3 <= L; ++l3) {
      int p = 0;
#pragma unroll
      for (int l1 = 0; l1 <= L; ++l1)
#pragma unroll
        for (int l2 = 0; l2 <= L; ++l2)
          if (l3 >= (l1 > l2 ? l1 - l2 : l2 - l1) && l3 <= l1 + l2 && ((l1 + l2 + l3) & 1) == 0) ++p;
      Pl[l3] = p;
      zoff[l3] = o;
      o += (2 * l3 + 1) * p;
    }
  }
  const int n0 = blockIdx.x * kVChunk;
  const int n1 = min(N, n0 + kVChunk);
  for (int n = n0; n < n1; ++n) {
    const size_t base = (size_t)n * TP::NY * C + k;
    const float* gb = Bbar + (size_t)n * TP::ZROW * C + k;
    float a[TP::NY], b[TP::NY], ab[TP::NY], bb[TP::NY];
#pragma unroll
    for (int i = 0; i < TP::NY; ++i) {
      a[i] = __ldg(phi + base + (size_t)i * C);
      b[i] = __ldg(A + base + (size_t)i * C);
      ab[i] = __ldg(gz + base + (size_t)i * C);
      bb[i] = Abar[base + (size_t)i * C];
    }
    TP::vjp_paths(a, b, [&](int l3, int c, int eta) {
      return __ldg(gb + (size_t)(zoff[l3] + c * Pl[l3] + eta) * C);
    }, ab, bb);
#pragma unroll
    for (int i = 0; i < TP::NY; ++i) {
      pbn[base + (size_t)i * C] = ab[i];
      Abar[base + (size_t)i * C] = bb[i];
    }
  }
}

template <int L>
int launch_full_tp_vjp(int N, int C, const float* phi, const float* A, const float* Bbar,
                       const float* gz, float* pbn, float* Abar, cudaStream_t s) {
  dim3 grid((N + kVChunk - 1) / kVChunk, (C + 127) / 128);
  full_tp_vjp_kernel<L><<<grid, 128, 0, s>>>(N, C, phi, A, Bbar, gz, pbn, Abar);
  return cudaGetLastError() == cudaSuccess ? FC_OK : FC_ERR_CUDA;
}

int full_tp_vjp_dispatch(int L, int N, int C, const float* phi, const float* A, const float* Bbar,
                         const float* gz, float* pbn, float* Abar, cudaStream_t s) {
  switch (L) {
    case 1: return launch_full_tp_vjp<1>(N, C, phi, A, Bbar, gz, pbn, Abar, s);
    case 2: return launch_full_tp_vjp<2>(N, C, phi, A, Bbar, gz, pbn, Abar, s);
    case 3: return launch_full_tp_vjp<3>(N, C, phi, A, Bbar, gz, pbn, Abar, s);
    case 4: return launch_full_tp_vjp<4>(N, C, phi, A, Bbar, gz, pbn, Abar, s);
  }
  return FC_ERR_UNSUPPORTED_RANK;
}

// products of one step in the convolution's output layout (fc_full_ladder.cu)
template <int L>
__global__ void __launch_bounds__(128) full_tp_zrow_kernel(int N, int C, const float* __restrict__ phi,
                                                           const float* __restrict__ A,
                                                           float* __restrict__ Bz) {
  using TP = LadderTP<L>;
  const int k = blockIdx.y * blockDim.x + threadIdx.x;
  if (k >= C) return;
  const int n0 = blockIdx.x * kVChunk;
  const int n1 = min(N, n0 + kVChunk);
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

int full_tp_zrow_dispatch(int L, int N, int C, const float* phi, const float* A, float* Bz,
                          cudaStream_t s) {
  dim3 grid((N + kVChunk - 1) / kVChunk, (C + 127) / 128);
  switch (L) {
    case 1: full_tp_zrow_kernel<1><<<grid, 128, 0, s>>>(N, C, phi, A, Bz); break;
    case 2: full_tp_zrow_kernel<2><<<grid, 128, 0, s>>>(N, C, phi, A, Bz); break;
    case 3: full_tp_zrow_kernel<3><<<grid, 128, 0, s>>>(N, C, phi, A, Bz); break;
    case 4: full_tp_zrow_kernel<4><<<grid, 128, 0, s>>>(N, C, phi, A, Bz); break;
    default: return FC_ERR_UNSUPPORTED_RANK;
  }
  return cudaGetLastError() == cudaSuccess ? FC_OK : FC_ERR_CUDA;
}

void rank_path_counts(int L, int* Pl) {
  for (int l3 = 0; l3 <= L; ++l3) {
    Pl[l3] = 0;
    for (int l1 = 0; l1 <= L; ++l1)
      for (int l2 = 0; l2 <= L; ++l2)
        if (l3 >= (l1 > l2 ? l1 - l2 : l2 - l1) && l3 <= l1 + l2 && ((l1 + l2 + l3) & 1) == 0) ++Pl[l3];
  }
}

RowLayout node_layout(int L) {
  RowLayout g{};
  g.stride = (L + 1) * (L + 1);
  for (int l = 0; l <= L && l < 5; ++l) {
    g.off[l] = l * l;
    g.cmul[l] = 1;
  }
  return g;
}

RowLayout path_layout(int L, const int* Pl) {
  RowLayout g{};
  g.stride = out_row(L, 0);
  int o = 0;
  for (int l = 0; l <= L && l < 5; ++l) {
    g.off[l] = o;
    g.cmul[l] = Pl[l];
    o += (2 * l + 1) * Pl[l];
  }
  return g;
}

template <bool ACC>
int launch_rows_gemm(int N, int C, int L, const RowLayout& ai, const RowLayout& ao, const float* in,
                     const float* Bm, const long long* boff, float* out, cudaStream_t s) {
  int wmax = 0;
  for (int l = 0; l <= L; ++l) wmax = ao.wid[l] > wmax ? ao.wid[l] : wmax;
  const int Rmax = N * (2 * L + 1);
  dim3 grid((Rmax + kVBM - 1) / kVBM, (wmax + kVBN - 1) / kVBN, L + 1);
  rows_gemm_kernel<ACC><<<grid, 256, 0, s>>>(N, C, L, ai, ao, in, Bm, boff[0], boff[1],
                                             boff[2], boff[3], boff[4], out);
  return cudaGetLastError() == cudaSuccess ? FC_OK : FC_ERR_CUDA;
}

int launch_rows_wgrad(int N, int C, int L, const RowLayout& la, const RowLayout& lb, const float* a,
                      const float* b, float* Wb, const long long* woff, cudaStream_t s) {
  int wmax = 0;
  for (int l = 0; l <= L; ++l) wmax = lb.wid[l] > wmax ? lb.wid[l] : wmax;
  const int Rmax = N * (2 * L + 1);
  const int tiles = ((C + kVBM - 1) / kVBM) * ((wmax + kVBN - 1) / kVBN);
  dim3 grid((Rmax + kVRows - 1) / kVRows, tiles, L + 1);
  rows_wgrad_kernel<<<grid, 256, 0, s>>>(N, C, L, la, lb, a, b, Wb, woff[0], woff[1], woff[2],
                                         woff[3], woff[4]);
  return cudaGetLastError() == cudaSuccess ? FC_OK : FC_ERR_CUDA;
}

int check_full_vjp_desc(const fc_ladder_desc* d) {
  if (!d) return FC_ERR_ARG;
  if (d->channels <= 0 || d->order < 1 || d->lmax < 0) return FC_ERR_ARG;
  if (d->lmax < 1 || d->lmax > 4) return FC_ERR_UNSUPPORTED_RANK;
  if (d->channels % 4) return FC_ERR_ALIGN;
  return FC_OK;
}

}  // namespace
}  // namespace fc

using namespace fc;

// Tensor-core geometry of B_bar = p_bar Wq_l at C = 128: the rows of p_bar as
// FP32 component-major tiles (K = 128, k_l = 4) and P_l maps per rank, one per
// path, each writing its path's slot of the convolution's output layout.
static PathGeom bbar_geom(int L, int N) {
  int Pl[6] = {0, 0, 0, 0, 0, 0};
  rank_path_counts(L, Pl);
  const int kc[5] = {4, 4, 4, 4, 4};
  return path_geom_maps(L, N, kc, Pl);
}

extern "C" size_t fc_full_ladder_vjp_workspace_size(const fc_ladder_desc* d, int n_nodes) {
  if (check_full_vjp_desc(d) != FC_OK || n_nodes < 0) return 0;
  const size_t plane = (size_t)n_nodes * (d->lmax + 1) * (d->lmax + 1) * d->channels;
  const size_t zplane = (size_t)n_nodes * out_row(d->lmax, 0) * d->channels;
  // two running gradients; one step's products and their gradient
  size_t f = 2 * plane + (d->order > 1 ? 2 * zplane : 0);
  // tensor cores: p_bar as operand tiles and one step's split maps
  if (d->order > 1 && mix_tc_supported(d->lmax, d->channels)) {
    const PathGeom g = bbar_geom(d->lmax, n_nodes);
    f += (size_t)(pg_xbase(g, g.L + 1) + pg_wbase(g, g.L + 1));
  }
  return sizeof(float) * f;
}

extern "C" int fc_full_ladder_vjp(const fc_ladder_desc* d, int n_nodes, const float* A, const float* W1,
                                  const float* Wq, const float* states, const float* gz, float* A_bar,
                                  float* W1_bar, float* Wq_bar, void* workspace, size_t ws_bytes,
                                  fc_stream_t stream) {
  int st = check_full_vjp_desc(d);
  if (st != FC_OK) return st;
  if (n_nodes < 0) return FC_ERR_ARG;
  const int L = d->lmax, C = d->channels, order = d->order;
  if (!W1 || !W1_bar || (order > 1 && (!Wq || !Wq_bar))) return FC_ERR_ARG;
  if (!aligned16(W1) || !aligned16(W1_bar) || (order > 1 && (!aligned16(Wq) || !aligned16(Wq_bar))))
    return FC_ERR_ALIGN;
  const int P = num_paths(L);
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemsetAsync(W1_bar, 0, sizeof(float) * (size_t)(L + 1) * C * C, s) != cudaSuccess ||
      (order > 1 &&
       cudaMemsetAsync(Wq_bar, 0, sizeof(float) * (size_t)(order - 1) * C * P * C, s) != cudaSuccess))
    return FC_ERR_CUDA;
  if (n_nodes == 0) return FC_OK;
  if (!A || !states || !gz || !A_bar) return FC_ERR_ARG;
  if (!aligned16(A) || !aligned16(states) || !aligned16(gz) || !aligned16(A_bar)) return FC_ERR_ALIGN;
  const size_t need = fc_full_ladder_vjp_workspace_size(d, n_nodes);
  if (!workspace || ws_bytes < need) return FC_ERR_WORKSPACE;
  if (!aligned16(workspace)) return FC_ERR_ALIGN;

  const int NY = (L + 1) * (L + 1);
  const size_t plane = (size_t)n_nodes * NY * C;
  const size_t zplane = (size_t)n_nodes * out_row(L, 0) * C;
  float* pb = static_cast<float*>(workspace);
  float* pbn = pb + plane;
  float* Bq = pbn + plane;
  float* Bbar = Bq + zplane;
  const bool tc = order > 1 && mix_tc_supported(L, C);
  const PathGeom gb = bbar_geom(L, n_nodes);
  float* xs = Bbar + zplane;                      // tensor cores: p_bar tiles
  float* wsm = tc ? xs + pg_xbase(gb, gb.L + 1) : nullptr;   // and the split maps
  int Pl[6] = {0, 0, 0, 0, 0, 0};
  rank_path_counts(L, Pl);
  RowLayout nl = node_layout(L), pl = path_layout(L, Pl);
  for (int l = 0; l <= L; ++l) {
    nl.wid[l] = C;
    pl.wid[l] = Pl[l] * C;
  }
  // per-rank offsets of the [C][P_l C] blocks of one step's map, and of W1's [C][C]
  long long qoff[5] = {0, 0, 0, 0, 0}, w1off[5] = {0, 0, 0, 0, 0};
  {
    long long o = 0;
    for (int l = 0; l <= L; ++l) {
      qoff[l] = o;
      o += (long long)C * Pl[l] * C;
      w1off[l] = (long long)l * C * C;
    }
  }
  if (cudaMemsetAsync(A_bar, 0, sizeof(float) * plane, s) != cudaSuccess ||
      cudaMemcpyAsync(pb, gz, sizeof(float) * plane, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return FC_ERR_CUDA;
  // Wq_bar's operands for the tensor cores: p_bar in the node layout, B_q in the path slots
  WgGeom wq{n_nodes, L, nl.stride, pl.stride};
  wq.ob0 = pl.off[0], wq.ob1 = pl.off[1], wq.ob2 = pl.off[2], wq.ob3 = pl.off[3], wq.ob4 = pl.off[4];
  wq.pe0 = Pl[0], wq.pe1 = Pl[1], wq.pe2 = Pl[2], wq.pe3 = Pl[3], wq.pe4 = Pl[4];
  wq.wo0 = (int)qoff[0], wq.wo1 = (int)qoff[1], wq.wo2 = (int)qoff[2], wq.wo3 = (int)qoff[3], wq.wo4 = (int)qoff[4];
  const size_t wq_step = (size_t)C * P * C;
  for (int q = order; q >= 2; --q) {
    const float* phi_prev = states + (size_t)(q - 2) * plane;
    const float* Wqq = Wq + (size_t)(q - 2) * wq_step;
    float* Wqb = Wq_bar + (size_t)(q - 2) * wq_step;
    if ((st = full_tp_zrow_dispatch(L, n_nodes, C, phi_prev, A, Bq, s)) != FC_OK) return st;
    if (tc) {   // Wq_bar and B_bar on tcgen05 (three-term TF32 split), B_bar one map per path
      if ((st = launch_rows_wgrad_tc(wq, pb, Bq, Wqb, s)) != FC_OK ||
          (st = launch_path_split_rows(gb, pb, xs, s)) != FC_OK ||
          (st = launch_path_split_map_t(gb, Wqq, wsm, s)) != FC_OK ||
          (st = launch_path_mix_tc(gb, xs, wsm, Bbar, s)) != FC_OK)
        return st;
    } else if ((st = launch_rows_wgrad(n_nodes, C, L, nl, pl, pb, Bq, Wqb, qoff, s)) != FC_OK ||
               (st = launch_rows_gemm<false>(n_nodes, C, L, nl, pl, pb, Wqq, qoff, Bbar, s)) != FC_OK) {
      return st;
    }
    if ((st = full_tp_vjp_dispatch(L, n_nodes, C, phi_prev, A, Bbar, gz, pbn, A_bar, s)) != FC_OK)
      return st;
    float* t = pb;
    pb = pbn;
    pbn = t;
  }
  // the first map: W1_bar_l += pbar^T A, A_bar += pbar W1_l
  if ((st = mix_tc_supported(L, C) ? launch_rows_wgrad_tc(node_wg_geom(L, n_nodes), pb, A, W1_bar, s)
                                     : launch_rows_wgrad(n_nodes, C, L, nl, nl, pb, A, W1_bar, w1off, s)) != FC_OK ||
      (st = launch_rows_gemm<true>(n_nodes, C, L, nl, nl, pb, W1, w1off, A_bar, s)) != FC_OK)
    return st;
  return FC_OK;
}
