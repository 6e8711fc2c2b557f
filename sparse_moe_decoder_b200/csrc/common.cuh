// Internal helpers shared by the libzmoe kernels and host entry points.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include <string>

#include <nvtx3/nvToolsExt.h>

#include "zmoe.h"

namespace zmoe {

// ---------------------------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------------------------

// Records `msg` as this thread's last error and returns `st`.
zmoe_status fail(zmoe_status st, const std::string& msg);

// Clears this thread's last error.
void clear_error();

// After a launch: maps a pending CUDA error to ZMOE_ERR_CUDA.
zmoe_status check_launch(const char* what);

// Device address of this device's error counter (cached per device).
unsigned int* device_error_counter();

// Number of SMs of the current device (cached per device).
int num_sms();

// Maximum dynamic shared memory per block of the current device (opt-in size).
int max_smem_optin();

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline size_t dtype_size(zmoe_dtype dt) { return dt == ZMOE_BF16 ? 2 : 4; }

inline bool dtype_ok(int dt) { return dt == ZMOE_F32 || dt == ZMOE_BF16; }

// An NVTX range around one entry point, so that a profiler timeline shows each zmoe_* call
// (header-only NVTX v3: without a tool attached a push/pop costs a few nanoseconds).
struct TraceRange {
  explicit TraceRange(const char* name) { nvtxRangePushA(name); }
  ~TraceRange() { nvtxRangePop(); }
  TraceRange(const TraceRange&) = delete;
  TraceRange& operator=(const TraceRange&) = delete;
};
#define ZMOE_TRACE(name) ::zmoe::TraceRange zmoe_trace_range_(name)

#define ZMOE_REQUIRE(cond, msg)                                      \
  do {                                                               \
    if (!(cond)) return ::zmoe::fail(ZMOE_ERR_INVALID_ARG, (msg));   \
  } while (0)

// ---------------------------------------------------------------------------------------------
// device side
// ---------------------------------------------------------------------------------------------

__device__ __forceinline__ void record_device_error(unsigned int* counter) {
  if (counter) atomicAdd(counter, 1u);
}

__device__ __forceinline__ float bf16_to_f32(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// Round-to-nearest-even fp32 -> bf16 bits (cuda_bf16 intrinsic).
__device__ __forceinline__ uint16_t f32_to_bf16_bits(float v) {
  __nv_bfloat16 b = __float2bfloat16_rn(v);
  return *reinterpret_cast<uint16_t*>(&b);
}

// Unpacks 8 bf16 values held in a uint4 into fp32.
__device__ __forceinline__ void unpack_bf16x8(const uint4& v, float* out) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    out[2 * i] = __uint_as_float(w[i] << 16);
    out[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  return static_cast<uint32_t>(f32_to_bf16_bits(lo)) | (static_cast<uint32_t>(f32_to_bf16_bits(hi)) << 16);
}

// Streaming 16-byte global load that does not allocate in L1 (read-only data).
__device__ __forceinline__ uint4 ldg_stream(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

}  // namespace zmoe
