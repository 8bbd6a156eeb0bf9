// libflashcart: node-local correlation ladder and its VJP.
//
// FlashCart (arXiv 2610.06409) Sec. 5 Eq. (2) with path-reduced products
// (App. E "Path-reduced products") and a per-rank channel mix after every
// product:
//   B_v[n, l3, c, k] = sum_{paths (l1,l2)->l3} W_v[p, k] f_p(A_v[n,l1,:,k], A_1[n,l2,:,k])_c
//   A_{v+1}[n, l, c, :] = M_{v,l} B_v[n, l, c, :]        (C x C per rank)
//   z = A_1 + A_2 + ... + A_order
// Every product couples channel k only with channel k (channel-diagonal,
// Sec. 5), so the product kernel is one thread per channel walking a chunk
// of nodes with the path weights of its channel in registers.  The mix is a
// per-rank GEMM over the rows (node, component) of that rank: at C = 128 on
// the tcgen05 tensor cores with a three-term TF32 split (fc_mix_tc.cu), fed
// by a product kernel that writes its output pre-split in the mix's tiled
// layout, with z summed in one pass at the end; else the register-tiled FP32
// kernel below, which also adds the new state into z in its epilogue.  The VJP replays
// the steps backwards: B_v is recomputed, B_bar = M^T-product of A_bar,
// M_bar += A_bar^T B (split over row chunks, atomic tile adds), and the
// product VJP (App. C Eq. C1 per path) adds into A_v_bar and A_1_bar and
// accumulates W_bar over its node chunk before one atomic add per entry.
#include "fc_common.cuh"
#include "fc_device.cuh"
#include "fc_tc.cuh"
#include "generated/fc_ladder_L1.cuh"
#include "generated/fc_ladder_L2.cuh"
#include "generated/fc_ladder_L3.cuh"
#include "generated/fc_ladder_L4.cuh"

namespace fc {

// nodes per thread: the forward products take short chunks (more CTAs in
// flight to hide the memory latency); the product VJP keeps long ones because
// it adds its path-weight gradients atomically once per chunk
constexpr int kLadderFwdChunk = 4;
constexpr int kLadderNodeChunk = 8;

// ---------------------------------------------------------------------------
// channel-diagonal products
// ---------------------------------------------------------------------------
template <int L>
__global__ void __launch_bounds__(128) ladder_tp_kernel(int N, int C, const float* __restrict__ Av,
                                                        const float* __restrict__ A1,
                                                        const float* __restrict__ W,
                                                        float* __restrict__ B) {
  using TP = LadderTP<L>;
  const int k = blockIdx.y * blockDim.x + threadIdx.x;
  if (k >= C) return;
  float w[TP::P];
#pragma unroll
  for (int p = 0; p < TP::P; ++p) w[p] = __ldg(W + (size_t)p * C + k);
  const int n0 = blockIdx.x * kLadderFwdChunk;
  const int n1 = min(N, n0 + kLadderFwdChunk);
  for (int n = n0; n < n1; ++n) {
    const size_t base = (size_t)n * TP::NY * C + k;
    float a[TP::NY], b[TP::NY], o[TP::NY];
#pragma unroll
    for (int i = 0; i < TP::NY; ++i) {
      a[i] = __ldg(Av + base + (size_t)i * C);
      b[i] = __ldg(A1 + base + (size_t)i * C);
    }
    TP::fwd(a, b, w, o);
#pragma unroll
    for (int i = 0; i < TP::NY; ++i) B[base + (size_t)i * C] = o[i];
  }
}

// The same product written straight into the FP32 component-major tiles of
// the tensor-core map (PathGeom with k_l = CW / 32, CW = 128 or 256 channels):
// component c of rank l of node n is row n mod 128 of tile c nb + n / 128 of
// that rank.  A CTA
// takes 8 consecutive nodes x 32 consecutive channels: it first stages both
// operands (every component, as 16-byte cp.async copies: 8 per thread) in
// shared memory, rows padded to 36 floats so that the reads below hit 32
// distinct banks; then a warp takes the 8 nodes x 4 consecutive channels
// (one channel per thread), so each store of one component is one full
// 128-byte core matrix.
constexpr int kCmPad = 36;   // floats per staged (node, component) row of 32 channels

template <int L, int CW>
__global__ void __launch_bounds__(256, 2) ladder_tp_cm_kernel(PathGeom g, const float* __restrict__ Av,
                                                              const float* __restrict__ A1,
                                                              const float* __restrict__ W,
                                                              float* __restrict__ xs) {
  using TP = LadderTP<L>;
  constexpr int C = CW;
  constexpr int NY = TP::NY;
  extern __shared__ __align__(16) float sa[];   // [operand][component][node][kCmPad]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nb0 = 8 * blockIdx.x, k0 = 32 * blockIdx.y;
  // stage: (operand, component, node, 16-byte chunk) of the CTA's tile
  for (int q = threadIdx.x; q < 2 * NY * 8 * 8; q += 256) {
    const int ch = q & 7, nn = (q >> 3) & 7, r = q >> 6;
    const int op = r / NY, i = r - op * NY;
    const int n = nb0 + nn;
    const bool ok = n < g.N;
    const float* src = (op ? A1 : Av) + ((size_t)(ok ? n : 0) * NY + i) * C + k0 + 4 * ch;
    cp_async16(sa + ((op * NY + i) * 8 + nn) * kCmPad + 4 * ch, src, ok);
  }
  cp_async_commit();
  float w[TP::P];
  const int nn = lane >> 2, kk = 4 * warp + (lane & 3);
  const int n = nb0 + nn, k = k0 + kk;
#pragma unroll
  for (int p = 0; p < TP::P; ++p) w[p] = __ldg(W + (size_t)p * C + k);
  cp_async_wait<0>();
  __syncthreads();
  if (n >= g.N) return;
  float a[NY], b[NY], o[NY];
#pragma unroll
  for (int i = 0; i < NY; ++i) {
    a[i] = sa[(i * 8 + nn) * kCmPad + kk];
    b[i] = sa[((NY + i) * 8 + nn) * kCmPad + kk];
  }
  TP::fwd(a, b, w, o);
  const int cofs = (k >> 5) * 4096 + tc::core_offset(n & 127, k & 31, 128);
#pragma unroll
  for (int l = 0; l <= L; ++l) {
#pragma unroll
    for (int c = 0; c < 2 * l + 1; ++c)
      xs[pg_xbase(g, l) + (long long)(c * g.nb + (n >> 7)) * (CW / 32) * 4096 + cofs] = o[l * l + c];
  }
}

// Avbar += w VJP1, A1bar += w VJP2, Wbar += <g, f> (atomic, once per chunk).
// Avbar may alias A1bar (first step: A_v = A_1).
template <int L>
__global__ void __launch_bounds__(128) ladder_tp_vjp_kernel(int N, int C, const float* __restrict__ Av,
                                                            const float* __restrict__ A1,
                                                            const float* __restrict__ W,
                                                            const float* __restrict__ G,
                                                            float* Avbar, float* A1bar,
                                                            float* __restrict__ Wbar) {
  using TP = LadderTP<L>;
  const int k = blockIdx.y * blockDim.x + threadIdx.x;
  if (k >= C) return;
  float w[TP::P], wb[TP::P];
#pragma unroll
  for (int p = 0; p < TP::P; ++p) {
    w[p] = __ldg(W + (size_t)p * C + k);
    wb[p] = 0.0f;
  }
  const bool alias = (Avbar == A1bar);
  const int n0 = blockIdx.x * kLadderNodeChunk;
  const int n1 = min(N, n0 + kLadderNodeChunk);
  for (int n = n0; n < n1; ++n) {
    const size_t base = (size_t)n * TP::NY * C + k;
    // the running gradients are loaded with the inputs (one memory round trip
    // per node) and the products accumulate onto them
    float a[TP::NY], b[TP::NY], g[TP::NY], ab[TP::NY], bb[TP::NY];
#pragma unroll
    for (int i = 0; i < TP::NY; ++i) {
      a[i] = __ldg(Av + base + (size_t)i * C);
      b[i] = __ldg(A1 + base + (size_t)i * C);
      g[i] = __ldg(G + base + (size_t)i * C);
      bb[i] = A1bar[base + (size_t)i * C];
      ab[i] = alias ? 0.0f : Avbar[base + (size_t)i * C];
    }
    TP::vjp(a, b, w, g, ab, bb, wb);
    if (alias) {
#pragma unroll
      for (int i = 0; i < TP::NY; ++i) A1bar[base + (size_t)i * C] = ab[i] + bb[i];
    } else {
#pragma unroll
      for (int i = 0; i < TP::NY; ++i) {
        Avbar[base + (size_t)i * C] = ab[i];
        A1bar[base + (size_t)i * C] = bb[i];
      }
    }
  }
#pragma unroll
  for (int p = 0; p < TP::P; ++p) atomicAdd(Wbar + (size_t)p * C + k, wb[p]);
}

// ---------------------------------------------------------------------------
// per-rank channel mixing GEMMs (FP32, register-tiled)
// ---------------------------------------------------------------------------
// rows of rank l: i in [0, N(2l+1)) -> node n = i / (2l+1), component c.
__device__ __forceinline__ size_t rank_row(int i, int l, int NY, int C) {
  const int w = 2 * l + 1;
  const int n = i / w;
  const int c = i - n * w;
  return ((size_t)n * NY + l * l + c) * C;
}

enum { kMixFwd = 0, kMixBar = 1 };

constexpr int kBM = 64, kBN = 128, kBK = 32;

// kMixFwd: out[r][j] = sum_t in[r][t] M[j][t]   (in x M^T), z[r][j] += out
// kMixBar: out[r][j] = sum_t in[r][t] M[t][j]   (in x M)
template <int MODE>
__global__ void __launch_bounds__(256) ladder_mix_kernel(int N, int C, int NY,
                                                         const float* __restrict__ in,
                                                         const float* __restrict__ Mall,
                                                         float* __restrict__ out, float* z) {
  __shared__ __align__(16) float As[kBK][kBM + 4];
  __shared__ __align__(16) float Bs[kBK][kBN + 4];
  const int l = blockIdx.z;
  const int R = N * (2 * l + 1);
  const int r0 = blockIdx.x * kBM;
  if (r0 >= R) return;
  const int j0 = blockIdx.y * kBN;
  const float* M = Mall + (size_t)l * C * C;
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;  // 16 x 16 threads: 8 cols x 4 rows each
  float acc[4][8];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.0f;

  for (int t0 = 0; t0 < C; t0 += kBK) {
    // A tile: 64 rows x 32 t, two float4 per thread, stored t-major
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      const int idx = tid + s * 256;        // 0..511
      const int rr = idx >> 3, tq = (idx & 7) * 4;
      float4 v = zero4();
      if (r0 + rr < R && t0 + tq < C)
        v = __ldg(reinterpret_cast<const float4*>(in + rank_row(r0 + rr, l, NY, C) + t0 + tq));
      As[tq + 0][rr] = v.x; As[tq + 1][rr] = v.y; As[tq + 2][rr] = v.z; As[tq + 3][rr] = v.w;
    }
    // B tile: 32 t x 128 j
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      const int idx = tid + s * 256;        // 0..1023
      if (MODE == kMixFwd) {
        const int jj = idx >> 3, tq = (idx & 7) * 4;   // M[j][t..t+3]
        float4 v = zero4();
        if (j0 + jj < C && t0 + tq < C)
          v = __ldg(reinterpret_cast<const float4*>(M + (size_t)(j0 + jj) * C + t0 + tq));
        Bs[tq + 0][jj] = v.x; Bs[tq + 1][jj] = v.y; Bs[tq + 2][jj] = v.z; Bs[tq + 3][jj] = v.w;
      } else {
        const int tt = idx >> 5, jq = (idx & 31) * 4;  // M[t][j..j+3]
        float4 v = zero4();
        if (t0 + tt < C && j0 + jq < C)
          v = __ldg(reinterpret_cast<const float4*>(M + (size_t)(t0 + tt) * C + j0 + jq));
        *reinterpret_cast<float4*>(&Bs[tt][jq]) = v;
      }
    }
    __syncthreads();
#pragma unroll 8
    for (int t = 0; t < kBK; ++t) {
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
    const size_t base = rank_row(r, l, NY, C);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int j = j0 + tx * 8 + h * 4;
      if (j >= C) continue;
      const float4 v = make_float4(acc[i][h * 4], acc[i][h * 4 + 1], acc[i][h * 4 + 2], acc[i][h * 4 + 3]);
      *reinterpret_cast<float4*>(out + base + j) = v;
      if (MODE == kMixFwd) {
        float4 zz = *reinterpret_cast<float4*>(z + base + j);
        zz.x += v.x; zz.y += v.y; zz.z += v.z; zz.w += v.w;
        *reinterpret_cast<float4*>(z + base + j) = zz;
      }
    }
  }
}

constexpr int kWgradRows = 512;   // rows per CTA of the weight-gradient GEMM

// Mbar_l[k][j] += sum_{rows i of rank l} Abar[i][k] B[i][j]
__global__ void __launch_bounds__(256) ladder_wgrad_kernel(int N, int C, int NY,
                                                           const float* __restrict__ Abar,
                                                           const float* __restrict__ B,
                                                           float* __restrict__ Mbar) {
  __shared__ __align__(16) float As[kBK][kBM + 4];
  __shared__ __align__(16) float Bs[kBK][kBN + 4];
  const int l = blockIdx.z;
  const int R = N * (2 * l + 1);
  const int i0 = blockIdx.x * kWgradRows;
  if (i0 >= R) return;
  const int i1 = min(R, i0 + kWgradRows);
  const int ktiles = (C + kBM - 1) / kBM;
  const int k0 = (blockIdx.y % ktiles) * kBM;
  const int j0 = (blockIdx.y / ktiles) * kBN;
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  float acc[4][8];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.0f;
  for (int t0 = i0; t0 < i1; t0 += kBK) {
    // A: 32 rows x 64 k  (two float4 per thread)
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      const int idx = tid + s * 256;       // 0..511
      const int tt = idx >> 4, kq = (idx & 15) * 4;
      float4 v = zero4();
      if (t0 + tt < i1 && k0 + kq < C)
        v = __ldg(reinterpret_cast<const float4*>(Abar + rank_row(t0 + tt, l, NY, C) + k0 + kq));
      *reinterpret_cast<float4*>(&As[tt][kq]) = v;
    }
    // B: 32 rows x 128 j
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      const int idx = tid + s * 256;       // 0..1023
      const int tt = idx >> 5, jq = (idx & 31) * 4;
      float4 v = zero4();
      if (t0 + tt < i1 && j0 + jq < C)
        v = __ldg(reinterpret_cast<const float4*>(B + rank_row(t0 + tt, l, NY, C) + j0 + jq));
      *reinterpret_cast<float4*>(&Bs[tt][jq]) = v;
    }
    __syncthreads();
#pragma unroll 8
    for (int t = 0; t < kBK; ++t) {
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
  float* Ml = Mbar + (size_t)l * C * C;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int k = k0 + ty * 4 + i;
    if (k >= C) continue;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int jj = j0 + tx * 8 + j;
      if (jj < C) atomicAdd(Ml + (size_t)k * C + jj, acc[i][j]);
    }
  }
}

// z = A_1 + sum_v states[v], float4 per thread (plane % 4 == 0)
__global__ void __launch_bounds__(256) ladder_sum_kernel(size_t plane4, int S,
                                                         const float4* __restrict__ A1,
                                                         const float4* __restrict__ states,
                                                         float4* __restrict__ z) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < plane4;
       i += (size_t)gridDim.x * blockDim.x) {
    float4 acc = __ldg(A1 + i);
    for (int v = 0; v < S; ++v) {
      const float4 a = __ldcs(states + (size_t)v * plane4 + i);
      acc.x += a.x;
      acc.y += a.y;
      acc.z += a.z;
      acc.w += a.w;
    }
    __stcs(z + i, acc);
  }
}

static int launch_ladder_sum(size_t plane, int S, const float* A1, const float* states, float* z,
                             cudaStream_t s) {
  const size_t plane4 = plane / 4;
  const int grid = 8 * device_sm_count();
  ladder_sum_kernel<<<grid, 256, 0, s>>>(plane4, S, reinterpret_cast<const float4*>(A1),
                                         reinterpret_cast<const float4*>(states),
                                         reinterpret_cast<float4*>(z));
  return cudaGetLastError() == cudaSuccess ? FC_OK : FC_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// orchestration
// ---------------------------------------------------------------------------
static int check_ladder_desc(const fc_ladder_desc* d) {
  if (!d) return FC_ERR_ARG;
  if (d->channels <= 0 || d->order < 1 || d->lmax < 0) return FC_ERR_ARG;
  if (d->lmax < 1 || d->lmax > 4) return FC_ERR_UNSUPPORTED_RANK;
  if (d->channels % 4) return FC_ERR_ALIGN;
  return FC_OK;
}

// threads per block of the channel-diagonal kernels (one per channel): the
// channel count rounded up to a warp, at most 128, so narrow widths idle no
// more than a warp's remainder
static int tp_threads(int C) { return C >= 128 ? 128 : (C + 31) / 32 * 32; }

template <int L>
static int launch_tp(int N, int C, const float* Av, const float* A1, const float* W, float* B,
                     cudaStream_t s) {
  const int tb = tp_threads(C);
  dim3 grid((N + kLadderFwdChunk - 1) / kLadderFwdChunk, (C + tb - 1) / tb);
  ladder_tp_kernel<L><<<grid, tb, 0, s>>>(N, C, Av, A1, W, B);
  return cudaGetLastError() == cudaSuccess ? FC_OK : FC_ERR_CUDA;
}

template <int L>
static int launch_tp_vjp(int N, int C, const float* Av, const float* A1, const float* W,
                         const float* G, float* Avbar, float* A1bar, float* Wbar, cudaStream_t s) {
  const int tb = tp_threads(C);
  dim3 grid((N + kLadderNodeChunk - 1) / kLadderNodeChunk, (C + tb - 1) / tb);
  ladder_tp_vjp_kernel<L><<<grid, tb, 0, s>>>(N, C, Av, A1, W, G, Avbar, A1bar, Wbar);
  return cudaGetLastError() == cudaSuccess ? FC_OK : FC_ERR_CUDA;
}

static int tp_dispatch(int L, int N, int C, const float* Av, const float* A1, const float* W,
                       float* B, cudaStream_t s) {
  switch (L) {
    case 1: return launch_tp<1>(N, C, Av, A1, W, B, s);
    case 2: return launch_tp<2>(N, C, Av, A1, W, B, s);
    case 3: return launch_tp<3>(N, C, Av, A1, W, B, s);
    case 4: return launch_tp<4>(N, C, Av, A1, W, B, s);
  }
  return FC_ERR_UNSUPPORTED_RANK;
}

template <int L, int CW>
static int launch_tp_cm(const PathGeom& g, const float* Av, const float* A1, const float* W, float* xs,
                        cudaStream_t s) {
  const size_t smem = sizeof(float) * 2 * (L + 1) * (L + 1) * 8 * kCmPad;
  static DeviceFlags configured;
  if (set_smem_once(configured, ladder_tp_cm_kernel<L, CW>, smem) != FC_OK) return FC_ERR_CUDA;
  ladder_tp_cm_kernel<L, CW><<<dim3((g.N + 7) / 8, CW / 32), 256, smem, s>>>(g, Av, A1, W, xs);
  return cudaGetLastError() == cudaSuccess ? FC_OK : FC_ERR_CUDA;
}

static int tp_cm_dispatch(int L, int C, const PathGeom& g, const float* Av, const float* A1, const float* W,
                          float* xs, cudaStream_t s) {
  if (C == 256) {
    switch (L) {
      case 1: return launch_tp_cm<1, 256>(g, Av, A1, W, xs, s);
      case 2: return launch_tp_cm<2, 256>(g, Av, A1, W, xs, s);
      case 3: return launch_tp_cm<3, 256>(g, Av, A1, W, xs, s);
      case 4: return launch_tp_cm<4, 256>(g, Av, A1, W, xs, s);
      default: return FC_ERR_UNSUPPORTED_RANK;
    }
  }
  switch (L) {
    case 1: return launch_tp_cm<1, 128>(g, Av, A1, W, xs, s);
    case 2: return launch_tp_cm<2, 128>(g, Av, A1, W, xs, s);
    case 3: return launch_tp_cm<3, 128>(g, Av, A1, W, xs, s);
    case 4: return launch_tp_cm<4, 128>(g, Av, A1, W, xs, s);
    default: return FC_ERR_UNSUPPORTED_RANK;
  }
}

static int tp_vjp_dispatch(int L, int N, int C, const float* Av, const float* A1, const float* W,
                           const float* G, float* Avbar, float* A1bar, float* Wbar, cudaStream_t s) {
  switch (L) {
    case 1: return launch_tp_vjp<1>(N, C, Av, A1, W, G, Avbar, A1bar, Wbar, s);
    case 2: return launch_tp_vjp<2>(N, C, Av, A1, W, G, Avbar, A1bar, Wbar, s);
    case 3: return launch_tp_vjp<3>(N, C, Av, A1, W, G, Avbar, A1bar, Wbar, s);
    case 4: return launch_tp_vjp<4>(N, C, Av, A1, W, G, Avbar, A1bar, Wbar, s);
  }
  return FC_ERR_UNSUPPORTED_RANK;
}

template <int MODE>
static int launch_mix(int L, int N, int C, const float* in, const float* M, float* out, float* z,
                      cudaStream_t s) {
  const int NY = (L + 1) * (L + 1);
  const int Rmax = N * (2 * L + 1);
  dim3 grid((Rmax + kBM - 1) / kBM, (C + kBN - 1) / kBN, L + 1);
  ladder_mix_kernel<MODE><<<grid, 256, 0, s>>>(N, C, NY, in, M, out, z);
  return cudaGetLastError() == cudaSuccess ? FC_OK : FC_ERR_CUDA;
}

static int launch_wgrad(int L, int N, int C, const float* Abar, const float* B, float* Mbar,
                        cudaStream_t s) {
  const int NY = (L + 1) * (L + 1);
  const int Rmax = N * (2 * L + 1);
  const int tiles = ((C + kBM - 1) / kBM) * ((C + kBN - 1) / kBN);
  dim3 grid((Rmax + kWgradRows - 1) / kWgradRows, tiles, L + 1);
  ladder_wgrad_kernel<<<grid, 256, 0, s>>>(N, C, NY, Abar, B, Mbar);
  return cudaGetLastError() == cudaSuccess ? FC_OK : FC_ERR_CUDA;
}

}  // namespace fc

using namespace fc;

extern "C" {

int fc_ladder_num_paths(const fc_ladder_desc* d) {
  if (check_ladder_desc(d) != FC_OK) return -1;
  return num_paths(d->lmax);
}

// Tensor-core VJP scratch: a gradient in the tiled split layout plus one
// step's split mixing matrices.
static size_t tc_scratch_floats(int L, int N) {
  return mix_tc_operand_floats(L, N) + mix_tc_matrix_floats(L);
}

// Tensor-core forward at C = 128 or 256: the product as FP32 component-major
// tiles of K = C inputs (k_l = C / 32); at C = 256 each rank's 256 x 256
// matrix is two maps of 128 output channels (e_l = 2), and output row
// (n, c, e) of the map kernel is channels 128 e .. 128 e + 127 of node n's
// component c, the natural layout.
static bool fwd_tc(int L, int C) { return mix_tc_supported(L, 128) && (C == 128 || C == 256); }

static PathGeom fwd_geom(int L, int N, int C) {
  const int k = C / 32;
  const int kc[5] = {k, k, k, k, k};
  if (C == 128) return path_geom(L, N, kc);
  const int pe[5] = {2, 2, 2, 2, 2};
  return path_geom_maps(L, N, kc, pe);
}

size_t fc_product_ladder_workspace_size(const fc_ladder_desc* d, int n_nodes) {
  if (check_ladder_desc(d) != FC_OK || n_nodes < 0) return 0;
  const int NY = (d->lmax + 1) * (d->lmax + 1);
  if (fwd_tc(d->lmax, d->channels)) {
    const PathGeom g = fwd_geom(d->lmax, n_nodes, d->channels);
    return sizeof(float) * (size_t)(pg_xbase(g, g.L + 1) + pg_wbase(g, g.L + 1));
  }
  return sizeof(float) * (size_t)n_nodes * NY * d->channels;
}

int fc_product_ladder(const fc_ladder_desc* d, int n_nodes, const float* A1, const float* path_w,
                      const float* mix_w, float* states, float* z, void* workspace,
                      size_t ws_bytes, fc_stream_t stream) {
  int st = check_ladder_desc(d);
  if (st != FC_OK) return st;
  if (n_nodes < 0) return FC_ERR_ARG;
  if (n_nodes == 0) return FC_OK;
  const int L = d->lmax, C = d->channels, S = d->order - 1;
  if (!A1 || !z || (S > 0 && (!path_w || !mix_w || !states))) return FC_ERR_ARG;
  if (!aligned16(A1) || !aligned16(z) || (S > 0 && (!aligned16(mix_w) || !aligned4(path_w) ||
                                                    !aligned16(states))))
    return FC_ERR_ALIGN;
  const size_t need = fc_product_ladder_workspace_size(d, n_nodes);
  if (S > 0 && (!workspace || ws_bytes < need)) return FC_ERR_WORKSPACE;
  if (S > 0 && !aligned16(workspace)) return FC_ERR_ALIGN;
  cudaStream_t s = (cudaStream_t)stream;
  const int NY = (L + 1) * (L + 1);
  const size_t plane = (size_t)n_nodes * NY * C;
  const int P = num_paths(L);
  if (S > 0 && fwd_tc(L, C)) {
    // tensor cores: the product is written as FP32 component-major tiles,
    // the map kernel (K = 128 per rank, split to TF32 hi / lo in shared
    // memory) writes the states; z = A_1 + sum of the states at the end.
    // Rows past the last node of a tile are never written: the MMA column of
    // such a row depends on that row alone and is not stored.
    const PathGeom g = fwd_geom(L, n_nodes, C);
    float* xs = static_cast<float*>(workspace);
    float* wsm = xs + pg_xbase(g, L + 1);
    for (int v = 1; v <= S; ++v) {
      const float* Av = v == 1 ? A1 : states + (size_t)(v - 2) * plane;
      if ((st = tp_cm_dispatch(L, C, g, Av, A1, path_w + (size_t)(v - 1) * P * C, xs, s)) != FC_OK ||
          (st = launch_path_split_map(g, mix_w + (size_t)(v - 1) * (L + 1) * C * C, wsm, s)) != FC_OK ||
          (st = launch_path_mix_tc(g, xs, wsm, states + (size_t)(v - 1) * plane, s)) != FC_OK)
        return st;
    }
    return launch_ladder_sum(plane, S, A1, states, z, s);
  }
  if (cudaMemcpyAsync(z, A1, sizeof(float) * plane, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return FC_ERR_CUDA;
  float* B = static_cast<float*>(workspace);
  for (int v = 1; v <= S; ++v) {
    const float* Av = v == 1 ? A1 : states + (size_t)(v - 2) * plane;
    st = tp_dispatch(L, n_nodes, C, Av, A1, path_w + (size_t)(v - 1) * P * C, B, s);
    if (st != FC_OK) return st;
    st = launch_mix<kMixFwd>(L, n_nodes, C, B, mix_w + (size_t)(v - 1) * (L + 1) * C * C,
                             states + (size_t)(v - 1) * plane, z, s);
    if (st != FC_OK) return st;
  }
  return FC_OK;
}

size_t fc_product_ladder_vjp_workspace_size(const fc_ladder_desc* d, int n_nodes) {
  if (check_ladder_desc(d) != FC_OK || n_nodes < 0) return 0;
  const int NY = (d->lmax + 1) * (d->lmax + 1);
  size_t f = 4 * (size_t)n_nodes * NY * d->channels;
  // tensor cores: the split gradient and the matrices (for B_bar = A_bar M;
  // the weight gradient reads FP32 rows); at C = 256 the gradient as FP32
  // tiles of K = 256 and one step's two transposed maps per rank
  if (mix_tc_supported(d->lmax, d->channels)) {
    f += tc_scratch_floats(d->lmax, n_nodes);
  } else if (fwd_tc(d->lmax, d->channels)) {
    const PathGeom g = fwd_geom(d->lmax, n_nodes, d->channels);
    f += (size_t)(pg_xbase(g, g.L + 1) + pg_wbase(g, g.L + 1));
  }
  return sizeof(float) * f;
}

int fc_product_ladder_vjp(const fc_ladder_desc* d, int n_nodes, const float* A1,
                          const float* path_w, const float* mix_w, const float* states,
                          const float* gz, float* A1_bar, float* path_w_bar, float* mix_w_bar,
                          void* workspace, size_t ws_bytes, fc_stream_t stream) {
  int st = check_ladder_desc(d);
  if (st != FC_OK) return st;
  if (n_nodes < 0) return FC_ERR_ARG;
  const int L = d->lmax, C = d->channels, S = d->order - 1;
  const int NY = (L + 1) * (L + 1);
  const int P = num_paths(L);
  cudaStream_t s = (cudaStream_t)stream;
  if (!gz || !A1_bar || !A1) return FC_ERR_ARG;
  if (S > 0 && (!path_w || !mix_w || !states || !path_w_bar || !mix_w_bar)) return FC_ERR_ARG;
  if (!aligned16(A1) || !aligned16(gz) || !aligned16(A1_bar) ||
      (S > 0 && (!aligned16(mix_w) || !aligned16(states) || !aligned4(path_w) ||
                 !aligned4(path_w_bar) || !aligned4(mix_w_bar))))
    return FC_ERR_ALIGN;
  const size_t need = fc_product_ladder_vjp_workspace_size(d, n_nodes);
  if (S > 0 && n_nodes > 0 && (!workspace || ws_bytes < need)) return FC_ERR_WORKSPACE;
  if (S > 0 && n_nodes > 0 && !aligned16(workspace)) return FC_ERR_ALIGN;
  const size_t plane = (size_t)n_nodes * NY * C;
  if (S > 0) {
    if (cudaMemsetAsync(path_w_bar, 0, sizeof(float) * (size_t)S * P * C, s) != cudaSuccess ||
        cudaMemsetAsync(mix_w_bar, 0, sizeof(float) * (size_t)S * (L + 1) * C * C, s) != cudaSuccess)
      return FC_ERR_CUDA;
  }
  if (n_nodes == 0) return FC_OK;
  // every A_v feeds z directly
  if (cudaMemcpyAsync(A1_bar, gz, sizeof(float) * plane, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return FC_ERR_CUDA;
  float* ws = static_cast<float*>(workspace);
  float* B = ws;
  float* Bbar = ws + plane;
  float* Ab[2] = {ws + 2 * plane, ws + 3 * plane};
  const bool tc = mix_tc_supported(L, C);
  // C = 256: B_bar = A_bar M on the tcgen05 maps (the transposed matrix as two
  // maps of 128 output channels, K = 256); the weight gradient stays FP32 SIMT
  const bool tc256 = !tc && fwd_tc(L, C);
  const PathGeom g256 = tc256 ? fwd_geom(L, n_nodes, C) : PathGeom{};
  float* xs = ws + 4 * plane;                                   // tensor-core paths only
  float* wsm = tc ? xs + mix_tc_operand_floats(L, n_nodes) : tc256 ? xs + pg_xbase(g256, L + 1) : nullptr;
  const float* Anext_bar = gz;           // gradient of A_{v+1}
  for (int v = S; v >= 1; --v) {
    const float* Av = v == 1 ? A1 : states + (size_t)(v - 2) * plane;
    const float* W = path_w + (size_t)(v - 1) * P * C;
    const float* M = mix_w + (size_t)(v - 1) * (L + 1) * C * C;
    float* Avbar;
    if (v == 1) {
      Avbar = A1_bar;
    } else {
      Avbar = Ab[v & 1];
      if (cudaMemcpyAsync(Avbar, gz, sizeof(float) * plane, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
        return FC_ERR_CUDA;
    }
    float* Mbar = mix_w_bar + (size_t)(v - 1) * (L + 1) * C * C;
    if (tc) {
      // B_bar = A_bar M and M_bar += A_bar^T B on the tensor cores; B is recomputed
      if ((st = tp_dispatch(L, n_nodes, C, Av, A1, W, B, s)) != FC_OK ||
          (st = launch_mix_tc_split_rows(L, n_nodes, Anext_bar, xs, s)) != FC_OK ||
          (st = launch_mix_tc_split_matrix(1, L, M, wsm, s)) != FC_OK ||
          (st = launch_mix_tc(L, n_nodes, xs, wsm, Bbar, s)) != FC_OK ||
          (st = launch_rows_wgrad_tc(node_wg_geom(L, n_nodes), Anext_bar, B, Mbar, s)) != FC_OK)
        return st;
    } else if (tc256) {
      if ((st = tp_dispatch(L, n_nodes, C, Av, A1, W, B, s)) != FC_OK ||
          (st = launch_path_split_rows(g256, Anext_bar, xs, s)) != FC_OK ||
          (st = launch_path_split_map_t(g256, M, wsm, s)) != FC_OK ||
          (st = launch_path_mix_tc(g256, xs, wsm, Bbar, s)) != FC_OK ||
          (st = launch_wgrad(L, n_nodes, C, Anext_bar, B, Mbar, s)) != FC_OK)
        return st;
    } else {
      if ((st = tp_dispatch(L, n_nodes, C, Av, A1, W, B, s)) != FC_OK ||
          (st = launch_mix<kMixBar>(L, n_nodes, C, Anext_bar, M, Bbar, nullptr, s)) != FC_OK ||
          (st = launch_wgrad(L, n_nodes, C, Anext_bar, B, Mbar, s)) != FC_OK)
        return st;
    }
    if ((st = tp_vjp_dispatch(L, n_nodes, C, Av, A1, W, Bbar, Avbar, A1_bar,
                              path_w_bar + (size_t)(v - 1) * P * C, s)) != FC_OK)
      return st;
    Anext_bar = Avbar;
  }
  return FC_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// allocation-free variant of fc_product_ladder
// ---------------------------------------------------------------------------
// Some callers cannot allocate device memory: code that runs inside another
// framework's memory pool, where the pool already holds nearly all of HBM
// and a raw cudaMalloc fails or fragments it, and latency-critical loops,
// where cudaMalloc may synchronise the device.  For them the scratch of one
// product state lives in this fixed array, which every GPU that loads the
// library keeps until the process exits.  Host code must not use the
// array's name as a device address (it is a host-side stand-in); the device
// address comes from cudaGetSymbolAddress, once per device.
namespace fc {
constexpr size_t kLadderStaticScratchBytes = 16u << 20;   // 16 MiB per GPU
static __device__ __align__(256) float g_ladder_scratch[kLadderStaticScratchBytes / sizeof(float)];
static std::atomic<void*> g_ladder_scratch_addr[kMaxDevices];

// Device address of g_ladder_scratch on the current device (set-up on the
// first call per device), or nullptr if the runtime call fails.
static void* ladder_static_scratch() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  void* p = g_ladder_scratch_addr[dev].load(std::memory_order_acquire);
  if (p == nullptr) {
    if (cudaGetSymbolAddress(&p, g_ladder_scratch) != cudaSuccess) return nullptr;
    g_ladder_scratch_addr[dev].store(p, std::memory_order_release);
  }
  return p;
}
}  // namespace fc

extern "C" int fc_product_ladder_noalloc(const fc_ladder_desc* d, int n_nodes, const float* A1,
                                         const float* path_w, const float* mix_w, float* states,
                                         float* z, fc_stream_t stream) {
  int st = check_ladder_desc(d);
  if (st != FC_OK) return st;
  if (n_nodes < 0) return FC_ERR_ARG;
  const size_t need = fc_product_ladder_workspace_size(d, n_nodes);
  if (need > kLadderStaticScratchBytes) return FC_ERR_WORKSPACE;
  void* ws = ladder_static_scratch();
  if (ws == nullptr) return FC_ERR_CUDA;
  return fc_product_ladder(d, n_nodes, A1, path_w, mix_w, states, z, ws, need, stream);
}
