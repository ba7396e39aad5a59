// Pieces shared by the thin-factor kernels (k_thin.cu: register path and
// the r x r iteration; k_thin_bulk.cu: shared-memory staged path): the
// padded-rank configuration, the fp64 tensor-core MMA, the conditioning
// weight, vector element access and the factor geometry.
#pragma once

#include <cuda_bf16.h>

#include "dm_common.cuh"

namespace dm {
namespace thin {

constexpr int TT = 128;  // threads per CTA
constexpr int TW = TT / 32;

template <int RP>
struct TCfg {
  static constexpr bool MMA = RP >= 8;
  static constexpr int NB = MMA ? RP / 8 : 1;       // 8-row blocks
  static constexpr int KB = MMA ? RP / 4 : 1;       // 4-wide k steps
  static constexpr int NUB = NB * (NB + 1) / 2;     // upper-triangle 8x8 blocks
  static constexpr int PART = MMA ? NUB * 64 : RP * RP;  // doubles per Gram partial
  // padded r x r row of the iteration's shared matrices: RP + 4 doubles puts
  // the MMA fragment reads of 16 lanes on 16 distinct 8-byte bank pairs
  static constexpr int SLD = RP >= 16 ? RP + 4 : RP + 1;
  // long-side columns per slab (work unit of thin_gram / thin_apply)
  static constexpr int SLAB = RP <= 4 ? 2048 : RP <= 16 ? 512 : 1024;
  // the next step's loads are issued before the current step computes
  static constexpr bool DB = RP <= 16;
};

// D (8x8, two values per lane) += A (8x4) * B (4x8) in fp64.
// Lane l = 4g + t holds A[g][t], B[t][g], D[g][2t], D[g][2t+1].
__device__ __forceinline__ void dmma(double& d0, double& d1, double a, double b) {
  asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};"
               : "+d"(d0), "+d"(d1)
               : "d"(a), "d"(b));
}

// C_j^2 = (e_j / mean(e) + eps)^(-1/2); the same expression in every launch.
__device__ __forceinline__ float col_weight(float e, float inv_mean, float eps) {
  return rsqrtf(__fmaf_rn(e, inv_mean, eps));
}

// 4 consecutive elements at flat index i (aligned to 4 elements).
__device__ __forceinline__ void ld4(const void* p, int64_t i, int dt, float v[4]) {
  if (dt == DT_BF16) {
    const uint2 u = *reinterpret_cast<const uint2*>(reinterpret_cast<const __nv_bfloat16*>(p) + i);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
    const float2 a = __bfloat1622float2(h[0]), b = __bfloat1622float2(h[1]);
    v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
  } else {
    const float4 f = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(p) + i);
    v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
  }
}

__device__ __forceinline__ void st4(void* p, int64_t i, int dt, const float v[4]) {
  if (dt == DT_BF16) {
    uint2 u;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
    h[0] = __floats2bfloat162_rn(v[0], v[1]);
    h[1] = __floats2bfloat162_rn(v[2], v[3]);
    *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(p) + i) = u;
  } else {
    *reinterpret_cast<float4*>(reinterpret_cast<float*>(p) + i) = make_float4(v[0], v[1], v[2], v[3]);
  }
}

// Two consecutive elements (aligned to 2 elements).
__device__ __forceinline__ void ld2(const void* p, int64_t i, int dt, float& v0, float& v1) {
  if (dt == DT_BF16) {
    const float2 a = __bfloat1622float2(
        *reinterpret_cast<const __nv_bfloat162*>(reinterpret_cast<const __nv_bfloat16*>(p) + i));
    v0 = a.x; v1 = a.y;
  } else {
    const float2 f = *reinterpret_cast<const float2*>(reinterpret_cast<const float*>(p) + i);
    v0 = f.x; v1 = f.y;
  }
}

__device__ __forceinline__ void st2(void* p, int64_t i, int dt, float v0, float v1) {
  if (dt == DT_BF16)
    *reinterpret_cast<__nv_bfloat162*>(reinterpret_cast<__nv_bfloat16*>(p) + i) =
        __floats2bfloat162_rn(v0, v1);
  else
    *reinterpret_cast<float2*>(reinterpret_cast<float*>(p) + i) = make_float2(v0, v1);
}

// Factor geometry in the orientation of the iteration: r short-side rows,
// n long-side columns; element (i, j) sits at j * r + i (tall storage) or
// i * n + j (wide storage).
struct Geo {
  bool tall;
  int r;
  int64_t n;
  float* e_r;  // energies along the short side (r entries)
  float* e_c;  // energies along the long side (n entries)
  bool cond;
  bool vec;    // 4-element vector access is aligned
  __device__ __forceinline__ int64_t off(int i, int64_t j) const {
    return tall ? j * r + i : (int64_t)i * n + j;
  }
};

__device__ __forceinline__ Geo geometry(const ThinMat& mt, int conditioned) {
  Geo q;
  q.tall = mt.rows > mt.cols;
  q.r = (int)(q.tall ? mt.cols : mt.rows);
  q.n = q.tall ? mt.rows : mt.cols;
  q.e_r = q.tall ? mt.e_col : mt.e_row;
  q.e_c = q.tall ? mt.e_row : mt.e_col;
  q.cond = conditioned && q.e_r != nullptr && q.e_c != nullptr;
  // wide rows must start on 4-element boundaries; tall runs of four
  // long-side columns are 4r contiguous elements starting at a multiple of 4r
  q.vec = mt.vec && (q.tall || (q.n & 3) == 0);
  return q;
}


}  // namespace thin
}  // namespace dm
