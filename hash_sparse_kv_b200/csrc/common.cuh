// Device helpers shared by the kernels of the hash-code KV retrieval library.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "hkv.h"

namespace hkv {

constexpr int kHeadDim = 128;

// First device-side error wins; later ones are dropped.
__device__ __forceinline__ void report(int32_t* status, int32_t code) {
  if (status != nullptr) atomicCAS(status, 0, code);
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Streaming vector loads of read-once data (no L1 allocation).
__device__ __forceinline__ void ld_stream(const uint32_t* p, uint32_t (&v)[4]) {
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3])
               : "l"(p));
}
__device__ __forceinline__ void ld_stream(const uint32_t* p, uint32_t (&v)[2]) {
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(v[0]), "=r"(v[1]) : "l"(p));
}
__device__ __forceinline__ void ld_stream(const uint32_t* p, uint32_t (&v)[1]) {
  asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v[0]) : "l"(p));
}

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

// Four consecutive elements starting at p (p 8-byte aligned for bf16,
// 16-byte aligned for fp32), widened to fp32.
__device__ __forceinline__ float4 load4_f32(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ float4 load4_f32(const __nv_bfloat16* p) {
  uint2 raw = *reinterpret_cast<const uint2*>(p);
  __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162*>(&raw.x);
  __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162*>(&raw.y);
  float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
  return make_float4(fa.x, fa.y, fb.x, fb.y);
}

// Row addressing shared by the encoders: row r is member r % per_group of
// group r / per_group.
struct RowMap {
  int64_t rows, per_group;
  int64_t x_group, x_row;  // element strides of the input vectors
  int64_t c_group, c_row;  // word strides of the codes
  int64_t n_group, n_row;  // element strides of the norms
  // (one group -- every call from hkv_encode_keys -- needs no 64-bit division)
  __device__ __forceinline__ int64_t x_off(int64_t r) const {
    return per_group >= rows ? r * x_row : (r / per_group) * x_group + (r % per_group) * x_row;
  }
  __device__ __forceinline__ int64_t c_off(int64_t r) const {
    return per_group >= rows ? r * c_row : (r / per_group) * c_group + (r % per_group) * c_row;
  }
  __device__ __forceinline__ int64_t n_off(int64_t r) const {
    return per_group >= rows ? r * n_row : (r / per_group) * n_group + (r % per_group) * n_row;
  }
};

}  // namespace hkv
