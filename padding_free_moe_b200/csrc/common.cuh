// Shared device/host helpers of libpfmoe (internal; not part of the C ABI).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <string>

#include "../../include/pfmoe.h"

namespace pfmoe {

// ---------------------------------------------------------------- host status
// Thread-local last error; set by fail() and returned by moe_last_error().
void set_error(const std::string& msg);
int fail(int code, const std::string& msg);

// Kernel profiler hooks (no-ops unless moe_profile_enable(1)).
void prof_begin(const char* name, cudaStream_t s);
void prof_end(const char* name, cudaStream_t s);

// Launch check: returns PFMOE_ERR_CUDA with a message if the last launch failed.
int check_launch(const char* what);

int num_sms();

// Raise a kernel's dynamic shared-memory limit to `bytes` (at most the device's opt-in limit
// less the kernel's static shared memory) on the current device.  cudaFuncSetAttribute acts
// on the current device only, so this is done once per (device, kernel) pair; thread-safe.
// Every launch then requests no more than the bytes its plan computed from the same limit.
int smem_optin(const void* kernel, int bytes, const char* name);

#define PFMOE_TRY(expr)            \
  do {                             \
    int _rc = (expr);              \
    if (_rc != PFMOE_OK) return _rc; \
  } while (0)

// Wrap a kernel launch with the profiler and a launch check.
#define PFMOE_LAUNCH(name, stream, ...)        \
  do {                                         \
    ::pfmoe::prof_begin(name, stream);         \
    __VA_ARGS__;                               \
    ::pfmoe::prof_end(name, stream);           \
    PFMOE_TRY(::pfmoe::check_launch(name));    \
  } while (0)

// ------------------------------------------------------------- device helpers
template <typename T> struct Vec;  // 16-byte vector of T
template <> struct Vec<float> { static constexpr int n = 4; };
template <> struct Vec<__nv_bfloat16> { static constexpr int n = 8; };

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }
template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

// Load/store 16 bytes as float[Vec<T>::n].
template <typename T>
__device__ __forceinline__ void load16(const T* p, float* out) {
  uint4 u = *reinterpret_cast<const uint4*>(p);
  if constexpr (sizeof(T) == 4) {
    out[0] = __uint_as_float(u.x); out[1] = __uint_as_float(u.y);
    out[2] = __uint_as_float(u.z); out[3] = __uint_as_float(u.w);
  } else {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 f = __bfloat1622float2(h[i]);
      out[2 * i] = f.x; out[2 * i + 1] = f.y;
    }
  }
}

template <typename T>
__device__ __forceinline__ void store16(T* p, const float* in) {
  uint4 u;
  if constexpr (sizeof(T) == 4) {
    u.x = __float_as_uint(in[0]); u.y = __float_as_uint(in[1]);
    u.z = __float_as_uint(in[2]); u.w = __float_as_uint(in[3]);
  } else {
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(in[2 * i], in[2 * i + 1]);
  }
  *reinterpret_cast<uint4*>(p) = u;
}

__device__ __forceinline__ void dev_error(int32_t* err, int bits) {
  if (err) atomicOr(err, bits);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float silu_f(float u) { return u / (1.0f + expf(-u)); }

}  // namespace pfmoe
