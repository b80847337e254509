// Shared device helpers for the decode kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace dv {

constexpr int kWarp = 32;

// Programmatic dependent launch: a kernel launched with programmatic stream
// serialisation may start while its predecessor drains; it must wait before
// reading anything an earlier kernel wrote. Without the launch attribute both
// instructions are no-ops.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::); }

// 16-byte load of data that is streamed once per step (weights, KV), with
// the streaming cache hint. A coherent load on purpose: loads issued before
// griddep_wait() then overlap the previous kernel, which the read-only (.nc)
// path does not do (measured on B200: 2.3 vs 6.6 TB/s for a chain of
// 6.3 MB weight streams). Volatile, so the compiler keeps it where it is
// written relative to griddep_wait().
__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 r;
  asm volatile("ld.global.cs.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// 16-byte load through L2 only (data another CTA of the same grid wrote).
__device__ __forceinline__ float4 ld_cg4(const float* p) { return __ldcg(reinterpret_cast<const float4*>(p)); }

// Element traits: a 16-byte vector holds E elements of T.
template <typename T>
struct WT;

template <>
struct WT<float> {
  static constexpr int E = 4;
  __device__ static __forceinline__ void unpack(const uint4& u, float (&f)[4]) {
    f[0] = __uint_as_float(u.x);
    f[1] = __uint_as_float(u.y);
    f[2] = __uint_as_float(u.z);
    f[3] = __uint_as_float(u.w);
  }
  __device__ static __forceinline__ float store_cvt(float v) { return v; }
};

template <>
struct WT<__nv_bfloat16> {
  static constexpr int E = 8;
  // bf16 is the upper half of a binary32: element 2i sits in the low 16 bits.
  __device__ static __forceinline__ void unpack(const uint4& u, float (&f)[8]) {
    f[0] = __uint_as_float(u.x << 16);
    f[1] = __uint_as_float(u.x & 0xffff0000u);
    f[2] = __uint_as_float(u.y << 16);
    f[3] = __uint_as_float(u.y & 0xffff0000u);
    f[4] = __uint_as_float(u.z << 16);
    f[5] = __uint_as_float(u.z & 0xffff0000u);
    f[6] = __uint_as_float(u.w << 16);
    f[7] = __uint_as_float(u.w & 0xffff0000u);
  }
  __device__ static __forceinline__ __nv_bfloat16 store_cvt(float v) { return __float2bfloat16_rn(v); }
};

// Weight-only int8 rows (a per-row scale applied by the kernel): a 16-byte
// vector holds 16 signed bytes, element i in byte i.
//
// Conversion without the integer-to-float unit: flipping a byte's sign bit
// gives u = x + 128 in [0, 255]; placed in the low mantissa byte of 2^23
// (bit pattern 0x4B0000uu, one byte permute) it is exactly the float
// 2^23 + u, and subtracting 2^23 + 128 leaves x exactly. One permute and one
// add per element, both at full rate.
template <>
struct WT<int8_t> {
  static constexpr int E = 16;
  __device__ static __forceinline__ void unpack(const uint4& u, float (&f)[16]) {
    const uint32_t w[4] = {u.x ^ 0x80808080u, u.y ^ 0x80808080u, u.z ^ 0x80808080u, u.w ^ 0x80808080u};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[4 * i + 0] = __uint_as_float(__byte_perm(w[i], 0x4B000000u, 0x7650u)) - 8388736.f;
      f[4 * i + 1] = __uint_as_float(__byte_perm(w[i], 0x4B000000u, 0x7651u)) - 8388736.f;
      f[4 * i + 2] = __uint_as_float(__byte_perm(w[i], 0x4B000000u, 0x7652u)) - 8388736.f;
      f[4 * i + 3] = __uint_as_float(__byte_perm(w[i], 0x4B000000u, 0x7653u)) - 8388736.f;
    }
  }
};

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Sum over a block of NT threads; every thread gets the result. `red` holds
// at least NT/32 floats; the call ends with a barrier so `red` can be reused.
template <int NT>
__device__ __forceinline__ float block_sum(float v, float* red) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  v = warp_sum(v);
  if (lane == 0) red[w] = v;
  __syncthreads();
  float t = (lane < NT / 32) ? red[lane] : 0.f;
  t = warp_sum(t);
  __syncthreads();
  return t;
}

template <int NT>
__device__ __forceinline__ float block_max(float v, float* red) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  v = warp_max(v);
  if (lane == 0) red[w] = v;
  __syncthreads();
  float t = (lane < NT / 32) ? red[lane] : -INFINITY;
  t = warp_max(t);
  __syncthreads();
  return t;
}

// Exclusive prefix sum over a block of NT threads. Returns this thread's
// exclusive prefix; *total receives the block total. `sc` holds NT/32 ints.
template <int NT>
__device__ __forceinline__ unsigned block_exclusive_scan(unsigned v, unsigned* sc, unsigned* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  unsigned incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    unsigned t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) sc[w] = incl;
  __syncthreads();
  if (w == 0) {
    unsigned s = (lane < NT / 32) ? sc[lane] : 0u;
    unsigned si = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      unsigned t = __shfl_up_sync(0xffffffffu, si, o);
      if (lane >= o) si += t;
    }
    if (lane < NT / 32) sc[lane] = si - s;  // exclusive warp offsets
    if (lane == 31) sc[NT / 32] = si;        // total (sc holds NT/32 + 1)
  }
  __syncthreads();
  unsigned r = sc[w] + incl - v;
  *total = sc[NT / 32];
  __syncthreads();
  return r;
}

__device__ __forceinline__ void raise_status(int* st, int bit) { atomicOr(st, bit); }

// The MLP's activation sigma of eq. (1): ReLU, or GeLU in its exact form
// v Phi(v) = v (1 + erf(v / sqrt(2))) / 2 (erff is CUDA's error function).
enum : int { ACT_RELU = 0, ACT_GELU = 1 };
__device__ __forceinline__ float activate(float v, int act) {
  return act == ACT_GELU ? 0.5f * v * (1.f + erff(v * 0.70710678118654752f)) : fmaxf(v, 0.f);
}

// out[0..3] += v without returning the old values (a fire-and-forget vector
// reduction in L2, so the issuing thread does not wait for it).
__device__ __forceinline__ void red_add4(float* out, float4 v) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(out), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w)
               : "memory");
}

}  // namespace dv
