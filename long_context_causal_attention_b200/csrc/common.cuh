// Shared device helpers for liblwm_attn (CUDA, sm_100a).
#pragma once

#include <climits>

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "lwm_attn.h"

namespace lwm {

constexpr int kTile = 128;  // rows per query / key tile in every kernel

// Status word layout at the start of the workspace (256 bytes reserved).
struct DeviceStatus {
  int32_t code;       // lwm_status written by a kernel whose bounded wait ran out
  int32_t where;      // which wait gave up (kernel-defined tag)
  int32_t block;      // blockIdx.x of the reporting CTA
  int32_t item_counter[4];  // work-queue heads of the persistent kernels (zeroed per call)
  int32_t pad[57];
};
static_assert(sizeof(DeviceStatus) == 256, "status block is 256 bytes");

__device__ __forceinline__ void report_status(DeviceStatus* st, lwm_status code, int where) {
  if (st) {
    atomicCAS(&st->code, 0, (int)code);
    st->where = where;
    st->block = (int)blockIdx.x;
  }
}

__device__ __forceinline__ void report_timeout(DeviceStatus* st, int where) {
  if (st) {
    atomicCAS(&st->code, 0, (int)LWM_ERR_TIMEOUT);
    st->where = where;
    st->block = (int)blockIdx.x;
  }
}

// ---------------------------------------------------------------------------
// element conversion
// ---------------------------------------------------------------------------
template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// ---------------------------------------------------------------------------
// RoPE angle: p * w_t with w_t = theta^(-2t/D), formed and reduced modulo 2pi
// in fp64 (Cody-Waite reduction with 2pi split into a double and its
// remainder), then cos/sin in fp32.  At p ~ 1e6 an fp32 angle would carry an
// error of ~0.06 rad; the fp64 form keeps the reduced angle to ~1e-10.
// ---------------------------------------------------------------------------
constexpr double kTwoPiHi = 6.283185307179586;         // nearest double to 2*pi
constexpr double kTwoPiLo = 2.4492935982947064e-16;    // 2*pi - kTwoPiHi
constexpr double kInvTwoPi = 0.15915494309189535;      // 1/(2*pi)

__device__ __forceinline__ double rope_freq(int t, int head_dim, double log2_theta) {
  return exp2(-(2.0 * (double)t / (double)head_dim) * log2_theta);
}

__device__ __forceinline__ void rope_cos_sin_w(int64_t pos, double w, float* c, float* s) {
  const double a = (double)pos * w;
  const double k = rint(a * kInvTwoPi);
  double r = fma(-k, kTwoPiHi, a);
  r = fma(-k, kTwoPiLo, r);
  sincosf((float)r, s, c);
}

// Same angle, cos/sin from the fast hardware approximation.  The argument is
// already reduced to [-pi, pi], where its absolute error is below 1e-6; used
// where the result is rounded to bf16 right after (relative 2^-9).
__device__ __forceinline__ void rope_cos_sin_fast(int64_t pos, double w, float* c, float* s) {
  const double a = (double)pos * w;
  const double k = rint(a * kInvTwoPi);
  double r = fma(-k, kTwoPiHi, a);
  r = fma(-k, kTwoPiLo, r);
  __sincosf((float)r, s, c);
}

// Packing mask of one 32 x 32 block, built by a whole warp: lane c holds the
// segment id of column c (col_seg; a value no row holds, e.g. INT_MIN, for a
// column past the end), every lane the id of its own row (row_seg).  Bit c of
// the result is set iff column c belongs to this lane's segment.  One load per
// lane instead of 32, and one pass per distinct row id in the warp (one or
// two for contiguous packed segments).  All 32 lanes must call it.
__device__ __forceinline__ uint32_t warp_segment_bits(int32_t col_seg, int32_t row_seg) {
  uint32_t bits = 0, pending = 0xffffffffu;
  while (pending) {
    const int32_t v = __shfl_sync(0xffffffffu, row_seg, __ffs(pending) - 1);
    const uint32_t cols = __ballot_sync(0xffffffffu, col_seg == v);
    const uint32_t rows = __ballot_sync(0xffffffffu, row_seg == v);
    if (row_seg == v) bits = cols;
    pending &= ~rows;
  }
  return bits;
}

// Bits [lo, hi) of a 32-bit word, 0 <= lo, hi <= 32.
__device__ __forceinline__ uint32_t bit_range(int lo, int hi) {
  if (hi <= lo) return 0u;
  const uint32_t upto_hi = hi >= 32 ? 0xffffffffu : ((1u << hi) - 1u);
  const uint32_t below_lo = lo >= 32 ? 0xffffffffu : ((1u << lo) - 1u);
  return upto_hi & ~below_lo;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

}  // namespace lwm
