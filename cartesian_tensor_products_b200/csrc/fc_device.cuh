// Device helpers shared by the libflashcart kernels (sm_100a).
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

namespace fc {

// ---- float4 arithmetic: four channels per lane, same operation ----------
// Packed FP32x2 (sm_100 fma.rn.f32x2 / mul.rn.f32x2): two channels per
// instruction, round-to-nearest, same result as two scalar fmaf/fmul.
__device__ __forceinline__ float2 lo2(float4 a) { return make_float2(a.x, a.y); }
__device__ __forceinline__ float2 hi2(float4 a) { return make_float2(a.z, a.w); }
__device__ __forceinline__ float4 cat2(float2 a, float2 b) { return make_float4(a.x, a.y, b.x, b.y); }
__device__ __forceinline__ float4 mul4(float4 a, float4 b) {
  return cat2(__fmul2_rn(lo2(a), lo2(b)), __fmul2_rn(hi2(a), hi2(b)));
}
__device__ __forceinline__ float4 fma4(float4 a, float4 b, float4 c) {
  return cat2(__ffma2_rn(lo2(a), lo2(b), lo2(c)), __ffma2_rn(hi2(a), hi2(b), hi2(c)));
}
__device__ __forceinline__ float4 mul4s(float s, float4 b) {
  const float2 ss = make_float2(s, s);
  return cat2(__fmul2_rn(ss, lo2(b)), __fmul2_rn(ss, hi2(b)));
}
// pair operand (s, s) already duplicated in memory: no register shuffling
__device__ __forceinline__ float4 mul4p(float2 ss, float4 b) {
  return cat2(__fmul2_rn(ss, lo2(b)), __fmul2_rn(ss, hi2(b)));
}
__device__ __forceinline__ float4 fma4p(float2 ss, float4 b, float4 c) {
  return cat2(__ffma2_rn(ss, lo2(b), lo2(c)), __ffma2_rn(ss, hi2(b), hi2(c)));
}
__device__ __forceinline__ float4 fma4s(float s, float4 b, float4 c) {
  const float2 ss = make_float2(s, s);
  return cat2(__ffma2_rn(ss, lo2(b), lo2(c)), __ffma2_rn(ss, hi2(b), hi2(c)));
}
__device__ __forceinline__ float4 zero4() { return make_float4(0.f, 0.f, 0.f, 0.f); }
// sum over the four channels of a lane of a * b
__device__ __forceinline__ float dot4(float4 a, float4 b) {
  const float2 p = __ffma2_rn(hi2(a), hi2(b), __fmul2_rn(lo2(a), lo2(b)));
  return p.x + p.y;
}

// ---- memory ----------------------------------------------------------------
// node features: read-only, re-read by many receivers -> keep in L1/L2
__device__ __forceinline__ float4 ld_x4(const float* p) {
  return __ldg(reinterpret_cast<const float4*>(p));
}
// edge weights: streamed once -> do not keep in L1
__device__ __forceinline__ float4 ld_w4(const float* p) {
  float4 v;
  asm("ld.global.nc.L1::no_allocate.v4.f32 {%0,%1,%2,%3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "l"(p));
  return v;
}
// shared memory
__device__ __forceinline__ float4 ld_s4(const float* p) {
  return *reinterpret_cast<const float4*>(p);
}
__device__ __forceinline__ void st_f4(float* p, float a, float b, float c, float d) {
  *reinterpret_cast<float4*>(p) = make_float4(a, b, c, d);
}
// outputs: written once
__device__ __forceinline__ void st_z4(float* p, float4 v) {
  __stcs(reinterpret_cast<float4*>(p), v);
}
__device__ __forceinline__ void red_add4(float* p, float4 v) {
  atomicAdd(reinterpret_cast<float4*>(p), v);
}

// ---- radial envelope of an edge of length r: s(r) and ds/dr --------------
// env = 1: s = scale (cos(pi r / rc) + 1) / 2 for r < rc, 0 beyond;
// env = 0: s = 1.
__device__ __forceinline__ void edge_envelope(int env, float r, float rc, float scale, float& s,
                                              float& sp) {
  if (!env) {
    s = 1.0f;
    sp = 0.0f;
    return;
  }
  if (!(r < rc)) {
    s = 0.0f;
    sp = 0.0f;
    return;
  }
  float sn, cs;
  sincospif(r / rc, &sn, &cs);
  s = 0.5f * scale * (cs + 1.0f);
  sp = -0.5f * scale * (3.14159265358979f / rc) * sn;
}

// ---- asynchronous global -> shared copies (one 16-byte slice per lane) --
// ok == false writes 16 zero bytes and reads nothing from src.
__device__ __forceinline__ void cp_async16(float* dst_smem, const float* src, bool ok) {
  const unsigned d = (unsigned)__cvta_generic_to_shared(dst_smem);
  const int n = ok ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(d), "l"(src), "r"(n)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;\n" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

}  // namespace fc
