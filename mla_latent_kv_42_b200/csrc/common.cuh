// Shared device helpers: element types, packed loads, warp reductions, the device status word,
// and the RoPE angle. Every kernel of libmla is compiled in one translation unit (libmla.cu).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "mla.h"

namespace mla {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// First device-side error since the last mla_read_device_status (0 = none). Kernels record
// errors here instead of trapping; the first writer wins.
__device__ int g_status;

__device__ __forceinline__ void record_error(int code) { atomicCAS(&g_status, 0, code); }

// Programmatic dependent launch. The library's kernels are launched so that the next one may
// start while this one finishes: each kernel lets its dependents launch once it is resident
// (griddep_launch), and every thread waits for the kernels before it to complete, with their
// memory visible, before it touches any memory they may write (griddep_wait). Each CTA passes
// a griddep_wait before it exits, so completion stays ordered from kernel to kernel. Without
// the launch attribute both are no-ops.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename T> struct Pack;
template <> struct Pack<__nv_bfloat16> {
  using T2 = __nv_bfloat162;
  static __device__ __forceinline__ float2 f2(T2 v) { return __bfloat1622float2(v); }
  static __device__ __forceinline__ T2 make(float a, float b) { return __floats2bfloat162_rn(a, b); }
  static __device__ __forceinline__ float f(__nv_bfloat16 v) { return __bfloat162float(v); }
  static __device__ __forceinline__ __nv_bfloat16 one(float a) { return __float2bfloat16_rn(a); }
};
template <> struct Pack<__half> {
  using T2 = __half2;
  static __device__ __forceinline__ float2 f2(T2 v) { return __half22float2(v); }
  static __device__ __forceinline__ T2 make(float a, float b) { return __floats2half2_rn(a, b); }
  static __device__ __forceinline__ float f(__half v) { return __half2float(v); }
  static __device__ __forceinline__ __half one(float a) { return __float2half_rn(a); }
};

// Store helpers for fp32 or element-type outputs.
template <typename O> struct Out;
template <> struct Out<float> {
  static __device__ __forceinline__ void put(float* p, float v) { *p = v; }
};
template <> struct Out<__nv_bfloat16> {
  static __device__ __forceinline__ void put(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }
};
template <> struct Out<__half> {
  static __device__ __forceinline__ void put(__half* p, float v) { *p = __float2half_rn(v); }
};

// 8 consecutive elements (16 bytes) to fp32.
template <typename T>
__device__ __forceinline__ void unpack8(const uint4& v, float (&f)[8]) {
  using T2 = typename Pack<T>::T2;
  const T2* p = reinterpret_cast<const T2*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 x = Pack<T>::f2(p[i]);
    f[2 * i] = x.x;
    f[2 * i + 1] = x.y;
  }
}

__device__ __forceinline__ uint4 ldg16(const void* p) { return __ldg(reinterpret_cast<const uint4*>(p)); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// cos/sin of the RoPE angle of pair k at position pos: pos * theta_k, with theta_k from the
// caller's table when one is given (e.g. YaRN-scaled frequencies), else base^(-2k/d_rope). The
// angle is formed and reduced in double precision (an fp32 angle at position 131072 would be off
// by up to ~1e-2 rad); only the final cos/sin are rounded to fp32.
__device__ __forceinline__ double rope_inv_freq(int k, int d_rope, double base, const double* table) {
  return table != nullptr ? table[k] : pow(base, -2.0 * (double)k / (double)d_rope);
}
__device__ __forceinline__ void rope_cos_sin_at(int pos, double inv_freq, float& c, float& s) {
  double sd, cd;
  sincos((double)pos * inv_freq, &sd, &cd);
  c = (float)cd;
  s = (float)sd;
}
__device__ __forceinline__ void rope_cos_sin(int pos, int k, int d_rope, double base, const double* table, float& c,
                                             float& s) {
  rope_cos_sin_at(pos, rope_inv_freq(k, d_rope, base, table), c, s);
}

// Launch `kern` on `st` with programmatic stream serialization: it may begin while the
// previous kernel in the stream finishes (see griddep_wait / griddep_launch).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

}  // namespace mla
