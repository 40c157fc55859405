// common.cuh -- device helpers shared by the sm_100a kernels of libmsc.
//
// io tensors are f32 or bf16; all arithmetic is f32.  Loads of a lane's run of
// consecutive elements use 16-byte vector accesses when the run is aligned and
// in bounds, element accesses otherwise (ragged tails, odd row lengths).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace msc {

using bf16 = __nv_bfloat16;

constexpr float kLog2e = 1.4426950408889634f;

// 2^x with the SFU's ex2 instruction (PTX ex2.approx.ftz.f32).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// softplus(v) = log(1 + e^v); for v > 20 it equals v to f32 precision.
__device__ __forceinline__ float softplus(float v) { return v > 20.f ? v : log1pf(expf(v)); }

__device__ __forceinline__ float sigmoid(float v) { return 1.f / (1.f + expf(-v)); }

__device__ __forceinline__ float silu(float v) { return v * sigmoid(v); }

// d/dv silu(v) = s (1 + v (1 - s)), s = sigmoid(v)
__device__ __forceinline__ float dsilu(float v) {
  float s = sigmoid(v);
  return s * (1.f + v * (1.f - s));
}

// ---------------------------------------------------------------------------
// element conversion
// ---------------------------------------------------------------------------
__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(bf16 v) { return __bfloat162float(v); }

template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ bf16 from_f32<bf16>(float v) { return __float2bfloat16_rn(v); }

// unpack one 32-bit word holding two bf16 (low half first in memory)
__device__ __forceinline__ void unpack_bf16x2(uint32_t w, float &lo, float &hi) {
  lo = __uint_as_float(w << 16);
  hi = __uint_as_float(w & 0xffff0000u);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t l = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(lo));
  uint32_t h = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(hi));
  return l | (h << 16);
}

// ---------------------------------------------------------------------------
// run loads / stores: v[i] = p[t0 + i] for i < K, positions >= n read `fill`
// ---------------------------------------------------------------------------
enum class Cache { kStream, kKeep };

template <Cache C>
__device__ __forceinline__ uint4 ld16(const void *p) {
  if constexpr (C == Cache::kStream) return __ldcs(reinterpret_cast<const uint4 *>(p));
  else return __ldg(reinterpret_cast<const uint4 *>(p));
}

template <int K, Cache C = Cache::kStream>
__device__ __forceinline__ void load_run(const float *p, int64_t t0, int64_t n, bool vec,
                                         float (&v)[K], float fill) {
  static_assert(K % 4 == 0, "run length must be a multiple of 4");
  if (vec && t0 + K <= n) {
#pragma unroll
    for (int j = 0; j < K / 4; ++j) {
      uint4 r = ld16<C>(p + t0 + 4 * j);
      v[4 * j + 0] = __uint_as_float(r.x);
      v[4 * j + 1] = __uint_as_float(r.y);
      v[4 * j + 2] = __uint_as_float(r.z);
      v[4 * j + 3] = __uint_as_float(r.w);
    }
  } else {
#pragma unroll
    for (int i = 0; i < K; ++i) v[i] = (t0 + i < n) ? p[t0 + i] : fill;
  }
}

template <int K, Cache C = Cache::kStream>
__device__ __forceinline__ void load_run(const bf16 *p, int64_t t0, int64_t n, bool vec,
                                         float (&v)[K], float fill) {
  static_assert(K % 8 == 0, "bf16 run length must be a multiple of 8");
  if (vec && t0 + K <= n) {
#pragma unroll
    for (int j = 0; j < K / 8; ++j) {
      uint4 r = ld16<C>(p + t0 + 8 * j);
      unpack_bf16x2(r.x, v[8 * j + 0], v[8 * j + 1]);
      unpack_bf16x2(r.y, v[8 * j + 2], v[8 * j + 3]);
      unpack_bf16x2(r.z, v[8 * j + 4], v[8 * j + 5]);
      unpack_bf16x2(r.w, v[8 * j + 6], v[8 * j + 7]);
    }
  } else {
#pragma unroll
    for (int i = 0; i < K; ++i) v[i] = (t0 + i < n) ? __bfloat162float(p[t0 + i]) : fill;
  }
}

template <int K>
__device__ __forceinline__ void store_run(float *p, int64_t t0, int64_t n, bool vec,
                                          const float (&v)[K]) {
  if (vec && t0 + K <= n) {
#pragma unroll
    for (int j = 0; j < K / 4; ++j) {
      uint4 r = make_uint4(__float_as_uint(v[4 * j]), __float_as_uint(v[4 * j + 1]),
                           __float_as_uint(v[4 * j + 2]), __float_as_uint(v[4 * j + 3]));
      __stcs(reinterpret_cast<uint4 *>(p + t0 + 4 * j), r);
    }
  } else {
#pragma unroll
    for (int i = 0; i < K; ++i)
      if (t0 + i < n) p[t0 + i] = v[i];
  }
}

template <int K>
__device__ __forceinline__ void store_run(bf16 *p, int64_t t0, int64_t n, bool vec,
                                          const float (&v)[K]) {
  if (vec && t0 + K <= n) {
#pragma unroll
    for (int j = 0; j < K / 8; ++j) {
      uint4 r = make_uint4(pack_bf16x2(v[8 * j + 0], v[8 * j + 1]),
                           pack_bf16x2(v[8 * j + 2], v[8 * j + 3]),
                           pack_bf16x2(v[8 * j + 4], v[8 * j + 5]),
                           pack_bf16x2(v[8 * j + 6], v[8 * j + 7]));
      __stcs(reinterpret_cast<uint4 *>(p + t0 + 8 * j), r);
    }
  } else {
#pragma unroll
    for (int i = 0; i < K; ++i)
      if (t0 + i < n) p[t0 + i] = __float2bfloat16_rn(v[i]);
  }
}

// ---------------------------------------------------------------------------
// warp scans of the linear-recurrence monoid
//   (p, h) o (p', h') = (p p', p' h + h')   -- "earlier o later"
// ---------------------------------------------------------------------------
// Inclusive prefix over lanes 0..lane (lane order = time order); returns the
// exclusive prefix in (pe, he) -- identity (1, 0) for lane 0.
__device__ __forceinline__ void warp_scan_fwd(float p, float h, float &pe, float &he) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    float pu = __shfl_up_sync(0xffffffffu, p, off);
    float hu = __shfl_up_sync(0xffffffffu, h, off);
    if (lane >= off) {
      h = fmaf(p, hu, h);
      p = p * pu;
    }
  }
  pe = __shfl_up_sync(0xffffffffu, p, 1);
  he = __shfl_up_sync(0xffffffffu, h, 1);
  if (lane == 0) { pe = 1.f; he = 0.f; }
}

// Suffix (reverse-time) version for the adjoint: a lane's transform maps the
// carry entering from the right, mu_in, to mu_out = p * mu_in + m.  Returns
// the composition of all lanes strictly to the right of this lane.
__device__ __forceinline__ void warp_scan_rev(float p, float m, float &ps, float &ms) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    float pd = __shfl_down_sync(0xffffffffu, p, off);
    float md = __shfl_down_sync(0xffffffffu, m, off);
    if (lane + off < 32) {
      m = fmaf(p, md, m);
      p = p * pd;
    }
  }
  ps = __shfl_down_sync(0xffffffffu, p, 1);
  ms = __shfl_down_sync(0xffffffffu, m, 1);
  if (lane == 31) { ps = 1.f; ms = 0.f; }
}

}  // namespace msc
