// Device-side helpers shared by the libdimuon kernels: storage conversions,
// reductions, the device status word and bounded waits.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "dm_internal.h"

namespace dm {

// ---------------------------------------------------------------------------
// Storage conversions.  bf16 stores round to nearest even (the intrinsic
// __float2bfloat16_rn); all arithmetic is fp32 or wider.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float ld_elem(const void* p, int64_t i, int dt) {
  return dt == DT_BF16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[i])
                       : reinterpret_cast<const float*>(p)[i];
}

__device__ __forceinline__ void st_elem(void* p, int64_t i, int dt, float v) {
  if (dt == DT_BF16)
    reinterpret_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(v);
  else
    reinterpret_cast<float*>(p)[i] = v;
}

// Value after a round trip through the storage dtype.
__device__ __forceinline__ float round_to(float v, int dt) {
  return dt == DT_BF16 ? __bfloat162float(__float2bfloat16_rn(v)) : v;
}

// M_t = mu M_{t-1} + G: the exact value rounded once to the storage dtype
// ("Muon Optimizer 정리", Update rule, eq. (1)).  fp32 storage: one fused
// multiply-add rounds the exact value to nearest.  bf16 storage: the two
// directed-rounding FMAs bracket the exact value; when they differ, the one
// with an odd last bit is the value rounded to odd at fp32 precision, and
// with 16 more bits than bf16 one rounding of it to nearest-even bf16 is the
// correctly rounded exact value (rounding to odd keeps the sticky
// information a second rounding needs).
__device__ __forceinline__ float momentum_value(float mu, float mprev, float g, int dt) {
  if (dt != DT_BF16) return __fmaf_rn(mu, mprev, g);
  const float lo = __fmaf_rd(mu, mprev, g), hi = __fmaf_ru(mu, mprev, g);
  const float odd = (__float_as_uint(lo) & 1u) ? lo : hi;
  return __bfloat162float(__float2bfloat16_rn(lo == hi ? hi : odd));  // hi: +0 for an exact 0
}

// Squared Frobenius norms below this floor give a zero update (fp32 cannot
// normalise them: the reciprocal square overflows).
constexpr double NORM2_FLOOR = 1e-30;

// 8 consecutive elements (16-byte aligned for bf16, 32-byte for fp32).
__device__ __forceinline__ void ld8(const void* p, int64_t i, int dt, float v[8]) {
  if (dt == DT_BF16) {
    uint4 u = *reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(p) + i);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float2 f = __bfloat1622float2(h[q]);
      v[2 * q] = f.x;
      v[2 * q + 1] = f.y;
    }
  } else {
    const float4* f = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(p) + i);
    float4 a = f[0], b = f[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
}

__device__ __forceinline__ void st8(void* p, int64_t i, int dt, const float v[8]) {
  if (dt == DT_BF16) {
    uint4 u;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
    for (int q = 0; q < 4; ++q) h[q] = __floats2bfloat162_rn(v[2 * q], v[2 * q + 1]);
    *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p) + i) = u;
  } else {
    float4* f = reinterpret_cast<float4*>(reinterpret_cast<float*>(p) + i);
    f[0] = make_float4(v[0], v[1], v[2], v[3]);
    f[1] = make_float4(v[4], v[5], v[6], v[7]);
  }
}

// ---------------------------------------------------------------------------
// Reductions (fixed shapes and orders, so results are reproducible).
// ---------------------------------------------------------------------------
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Block-wide sum; every thread gets the result.  `scratch` holds >= 32 floats.
__device__ __forceinline__ float block_sum(float v, float* scratch) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int nw = (blockDim.x + 31) >> 5;
  v = warp_sum(v);
  __syncthreads();
  if (lane == 0) scratch[wid] = v;
  __syncthreads();
  float t = 0.f;
  for (int w = 0; w < nw; ++w) t += scratch[w];
  return t;
}

__device__ __forceinline__ double block_sum_d(double v, double* scratch) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int nw = (blockDim.x + 31) >> 5;
  v = warp_sum_d(v);
  __syncthreads();
  if (lane == 0) scratch[wid] = v;
  __syncthreads();
  double t = 0.0;
  for (int w = 0; w < nw; ++w) t += scratch[w];
  return t;
}

// ---------------------------------------------------------------------------
// Device status word (first int32 of the workspace).  Codes only grow, so the
// most severe condition of a step survives.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void raise_status(int* status, int code) {
  if (status) atomicMax(status, code);
}

// A bounded wait that gave up also sets the abort word (the int32 after the
// status word).  Every later launch of the step reads it at its start and
// returns without writing, so no weight is updated from buffers that a
// timed-out launch left half written.
__device__ __forceinline__ void raise_timeout(int* status) {
  if (!status) return;
  atomicMax(status, ST_TIMEOUT);
  atomicExch(status + STATUS_ABORT_WORD, 1);
}

__device__ __forceinline__ bool step_aborted(const int* status) {
  return status && *reinterpret_cast<const volatile int*>(status + STATUS_ABORT_WORD) != 0;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Binary search: index g such that starts[g] <= x < starts[g + 1].
__device__ __forceinline__ int find_group(const int* starts, int count, int x) {
  int lo = 0, hi = count - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (starts[mid] <= x) lo = mid; else hi = mid - 1;
  }
  return lo;
}

}  // namespace dm
