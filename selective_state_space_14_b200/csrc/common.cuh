// common.cuh -- device helpers shared by the sm_100a kernels of libmsc.
//
// io tensors are f32, bf16 or f16; all arithmetic is f32.  Loads of a lane's run of
// consecutive elements use 16-byte vector accesses when the run is aligned and
// in bounds, element accesses otherwise (ragged tails, odd row lengths).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <type_traits>

namespace msc {

using bf16 = __nv_bfloat16;
using f16 = __half;

constexpr float kLog2e = 1.4426950408889634f;

// 2^x with the SFU's ex2 instruction (PTX ex2.approx.ftz.f32).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// softplus(v) = log(1 + e^v), e = e^v.  For e < 1/4, log(1 + e) is taken from
// the series of 2 atanh(s), s = e / (2 + e) <= 1/9 (log(1 + e) =
// log((1 + s) / (1 - s)) = 2 (s + s^3/3 + s^5/5 + ...); the terms kept leave a
// relative truncation error below s^10/11 < 3e-11), which keeps full relative
// accuracy for tiny e where log(1 + e) would cancel; otherwise 1 + e >= 1.25
// and the hardware logarithm is accurate.  For v > 20, softplus(v) = v in f32.
__device__ __forceinline__ float softplus(float v) {
  if (v > 20.f) return v;
  const float e = __expf(v);
  if (e < 0.25f) {
    const float s = __fdividef(e, 2.f + e);
    const float s2 = s * s;
    float r = fmaf(s2, 1.f / 9.f, 1.f / 7.f);
    r = fmaf(s2, r, 1.f / 5.f);
    r = fmaf(s2, r, 1.f / 3.f);
    r = fmaf(s2, r, 1.f);
    return 2.f * s * r;
  }
  return __logf(1.f + e);
}

// sin and cos of a cumulative angle: Cody and Waite's additive reduction by
// 2 pi, the constant split as 6.28125 (8 significant bits, so n * 6.28125 is
// exact for |n| < 2^16) plus the remainder 2 pi - 6.28125, then the SFU's sin
// and cos on [-pi, pi] (absolute error about 2^-21)
__device__ __forceinline__ void sincos_reduced(float phi, float &sn, float &cs) {
  const float n = rintf(phi * 0.15915494309189535f);
  float r = fmaf(-n, 6.28125f, phi);
  r = fmaf(-n, 1.9353071795864769e-3f, r);
  __sincosf(r, &sn, &cs);
}

// sigmoid(v) = 1 / (1 + e^-v), evaluated from e^-|v| so that it stays finite.
__device__ __forceinline__ float sigmoid(float v) {
  const float e = __expf(-fabsf(v));
  const float s = __fdividef(1.f, 1.f + e);
  return v >= 0.f ? s : e * s;
}

__device__ __forceinline__ float silu(float v) { return v * sigmoid(v); }

// d/dv silu(v) = s (1 + v (1 - s)), s = sigmoid(v)
__device__ __forceinline__ float dsilu(float v) {
  const float s = sigmoid(v);
  return s * (1.f + v * (1.f - s));
}

// ---------------------------------------------------------------------------
// packed pairs of f32 (PTX add/mul/fma .f32x2, sm_100+): one instruction
// computes two IEEE round-to-nearest results, bit-identical to two scalar ops
// ---------------------------------------------------------------------------
// Operands are packed into 64-bit registers inside the asm (mov.b64 {lo, hi}),
// so that no value is type-punned through memory.
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float2 splat2(float v) { return make_float2(v, v); }
__device__ __forceinline__ float2 ex2_2(float2 v) { return make_float2(ex2(v.x), ex2(v.y)); }

// ---------------------------------------------------------------------------
// element conversion
// ---------------------------------------------------------------------------
__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(bf16 v) { return __bfloat162float(v); }
__device__ __forceinline__ float to_f32(f16 v) { return __half2float(v); }

template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ bf16 from_f32<bf16>(float v) { return __float2bfloat16_rn(v); }
template <> __device__ __forceinline__ f16 from_f32<f16>(float v) { return __float2half_rn(v); }

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

// the same for either 16-bit io type (bf16 or f16)
template <typename T>
__device__ __forceinline__ void unpack2(uint32_t w, float &lo, float &hi) {
  if constexpr (std::is_same_v<T, bf16>) {
    unpack_bf16x2(w, lo, hi);
  } else {
    lo = __half2float(__ushort_as_half((unsigned short)(w & 0xffffu)));
    hi = __half2float(__ushort_as_half((unsigned short)(w >> 16)));
  }
}
template <typename T>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  if constexpr (std::is_same_v<T, bf16>) {
    return pack_bf16x2(lo, hi);
  } else {
    const uint32_t l = (uint32_t)__half_as_ushort(__float2half_rn(lo));
    const uint32_t h = (uint32_t)__half_as_ushort(__float2half_rn(hi));
    return l | (h << 16);
  }
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

template <int K, Cache C = Cache::kStream, typename T16>
__device__ __forceinline__ void load_run16(const T16 *p, int64_t t0, int64_t n, bool vec,
                                           float (&v)[K], float fill) {
  static_assert(K % 8 == 0, "16-bit run length must be a multiple of 8");
  if (vec && t0 + K <= n) {
#pragma unroll
    for (int j = 0; j < K / 8; ++j) {
      uint4 r = ld16<C>(p + t0 + 8 * j);
      unpack2<T16>(r.x, v[8 * j + 0], v[8 * j + 1]);
      unpack2<T16>(r.y, v[8 * j + 2], v[8 * j + 3]);
      unpack2<T16>(r.z, v[8 * j + 4], v[8 * j + 5]);
      unpack2<T16>(r.w, v[8 * j + 6], v[8 * j + 7]);
    }
  } else {
#pragma unroll
    for (int i = 0; i < K; ++i) v[i] = (t0 + i < n) ? to_f32(p[t0 + i]) : fill;
  }
}
template <int K, Cache C = Cache::kStream>
__device__ __forceinline__ void load_run(const bf16 *p, int64_t t0, int64_t n, bool vec,
                                         float (&v)[K], float fill) {
  load_run16<K, C>(p, t0, n, vec, v, fill);
}
template <int K, Cache C = Cache::kStream>
__device__ __forceinline__ void load_run(const f16 *p, int64_t t0, int64_t n, bool vec,
                                         float (&v)[K], float fill) {
  load_run16<K, C>(p, t0, n, vec, v, fill);
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

template <int K, typename T16>
__device__ __forceinline__ void store_run16(T16 *p, int64_t t0, int64_t n, bool vec,
                                            const float (&v)[K]) {
  if (vec && t0 + K <= n) {
#pragma unroll
    for (int j = 0; j < K / 8; ++j) {
      uint4 r = make_uint4(pack2<T16>(v[8 * j + 0], v[8 * j + 1]),
                           pack2<T16>(v[8 * j + 2], v[8 * j + 3]),
                           pack2<T16>(v[8 * j + 4], v[8 * j + 5]),
                           pack2<T16>(v[8 * j + 6], v[8 * j + 7]));
      __stcs(reinterpret_cast<uint4 *>(p + t0 + 8 * j), r);
    }
  } else {
#pragma unroll
    for (int i = 0; i < K; ++i)
      if (t0 + i < n) p[t0 + i] = from_f32<T16>(v[i]);
  }
}
template <int K>
__device__ __forceinline__ void store_run(bf16 *p, int64_t t0, int64_t n, bool vec,
                                          const float (&v)[K]) {
  store_run16<K>(p, t0, n, vec, v);
}
template <int K>
__device__ __forceinline__ void store_run(f16 *p, int64_t t0, int64_t n, bool vec,
                                          const float (&v)[K]) {
  store_run16<K>(p, t0, n, vec, v);
}

// ---------------------------------------------------------------------------
// asynchronous global -> shared copies (cp.async, 16 bytes; bytes past
// src_bytes are zero-filled).  Both addresses must be 16-byte aligned.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gmem_src, int src_bytes) {
  const uint32_t d = (uint32_t)__cvta_generic_to_shared(smem_dst);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(d), "l"(gmem_src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;\n" ::: "memory");
}
template <int kPending>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(kPending) : "memory");
}

// ---------------------------------------------------------------------------
// warp scan of the linear-recurrence monoid
//   (p, h) o (p', h') = (p p', p' h + h')   -- "earlier o later"
// (the combine of the Mamba-1 forward's time segments)
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

}  // namespace msc
