// Device helpers shared by the libflashcart kernels (sm_100a).
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

namespace fc {

// ---- float4 arithmetic: four channels per lane, same operation ----------
__device__ __forceinline__ float4 mul4(float4 a, float4 b) {
  return make_float4(a.x * b.x, a.y * b.y, a.z * b.z, a.w * b.w);
}
__device__ __forceinline__ float4 fma4(float4 a, float4 b, float4 c) {
  return make_float4(fmaf(a.x, b.x, c.x), fmaf(a.y, b.y, c.y),
                     fmaf(a.z, b.z, c.z), fmaf(a.w, b.w, c.w));
}
__device__ __forceinline__ float4 mul4s(float s, float4 b) {
  return make_float4(s * b.x, s * b.y, s * b.z, s * b.w);
}
__device__ __forceinline__ float4 fma4s(float s, float4 b, float4 c) {
  return make_float4(fmaf(s, b.x, c.x), fmaf(s, b.y, c.y), fmaf(s, b.z, c.z),
                     fmaf(s, b.w, c.w));
}
__device__ __forceinline__ float4 zero4() { return make_float4(0.f, 0.f, 0.f, 0.f); }

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

}  // namespace fc
