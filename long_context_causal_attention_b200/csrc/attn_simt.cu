// CUDA-core (SIMT, fp32 arithmetic) attention kernels.
//
// These serve the fp32 data type, where the answer must agree with the exact
// result to 1e-4 and tensor-core tf32 cannot, and head_dim 64.  One warp owns
// one query row (forward, dQ) or one key row (dK/dV); lanes split the head
// dimension for the value/gradient accumulators, and a group of 32 keys (or
// queries) is scored at once, one per lane.
//
// Math (LWM research note, "模型架构": exact blockwise attention with online
// softmax; "训练方法": packing mask; backward recomputes P from LSE as in the
// FlashAttention entry of the paper card's references):
//   forward   m, l running max / sum in log2 units, O = sum p v / l,
//             LSE = (m + log2 l) ln 2
//   dQ row i  dS_ij = P_ij (dO_i.v_j - D_i),  dq~_i = scale sum_j dS_ij k~_j
//   dK/dV j   dv_j = sum_i P_ij dO_i,  dk~_j = scale sum_i dS_ij q~_i
// Gradients are turned back from the rotated frame with R(p)^T in the
// epilogue (no separate pass, no atomics).
#include <cmath>

#include "common.cuh"
#include "internal.h"

namespace lwm {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr unsigned kFull = 0xffffffffu;

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int s = 16; s > 0; s >>= 1) x = fmaxf(x, __shfl_xor_sync(kFull, x, s));
  return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int s = 16; s > 0; s >>= 1) x += __shfl_xor_sync(kFull, x, s);
  return x;
}

// dot(smem fp32 row, global row of T) with 16-byte loads.
template <typename T, int D>
__device__ __forceinline__ float dot_row(const float* __restrict__ a, const T* __restrict__ row) {
  constexpr int N = 16 / sizeof(T);
  float acc = 0.f;
#pragma unroll
  for (int c = 0; c < D / N; ++c) {
    uint4 raw = __ldg(reinterpret_cast<const uint4*>(row) + c);
    const T* e = reinterpret_cast<const T*>(&raw);
#pragma unroll
    for (int u = 0; u < N; ++u) acc = fmaf(a[c * N + u], to_f32(e[u]), acc);
  }
  return acc;
}

__device__ __forceinline__ bool tile_may_hold(const int32_t* tmin, const int32_t* tmax, int64_t t,
                                              int32_t sid) {
  return !(tmin[t] > sid || tmax[t] < sid);
}

// R(pos)^T applied to this lane's DPL consecutive dims (DPL/2 pairs), in place.
template <int D>
__device__ __forceinline__ void unrotate_lane(float* x, int lane, int64_t pos, double log2_theta) {
  constexpr int DPL = D / 32;
#pragma unroll
  for (int u = 0; u < DPL / 2; ++u) {
    const int t = lane * (DPL / 2) + u;
    float c, s;
    rope_cos_sin_w(pos, rope_freq(t, D, log2_theta), &c, &s);
    const float a = x[2 * u], b = x[2 * u + 1];
    x[2 * u] = a * c + b * s;
    x[2 * u + 1] = b * c - a * s;
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(128)
simt_fwd_kernel(const T* __restrict__ qr, const T* __restrict__ kr, const T* __restrict__ v,
                T* __restrict__ o, float* __restrict__ lse, const int32_t* __restrict__ seg,
                const int32_t* __restrict__ kseg, const int32_t* __restrict__ ktmin,
                const int32_t* __restrict__ ktmax, int64_t S, int H, int64_t n_tiles,
                float scale_log2, int causal) {
  constexpr int DPL = D / 32;
  __shared__ float qs[4][D];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t i = (int64_t)blockIdx.x * 4 + warp;
  const int h = blockIdx.y;
  const int64_t b = blockIdx.z;
  if (i >= S) return;
  const size_t rs = (size_t)H * D;
  const size_t tok = (size_t)b * S + i;
  const T* qrow = qr + tok * rs + (size_t)h * D;
  for (int d = lane; d < D; d += 32) qs[warp][d] = to_f32(qrow[d]);
  __syncwarp();
  const int32_t si = seg ? seg[tok] : 0;
  float m = -INFINITY, l = 0.f, acc[DPL];
#pragma unroll
  for (int u = 0; u < DPL; ++u) acc[u] = 0.f;
  if (si >= 0) {
    const int64_t kend = causal ? i + 1 : S;
    for (int64_t t0 = 0; t0 < kend; t0 += kTile) {
      if (seg && !tile_may_hold(ktmin, ktmax, b * n_tiles + t0 / kTile, si)) continue;
      const int64_t t1 = min(t0 + (int64_t)kTile, kend);
      for (int64_t j0 = t0; j0 < t1; j0 += 32) {
        const int64_t j = j0 + lane;
        float s = -INFINITY;
        if (j < t1 && (!seg || kseg[(size_t)b * S + j] == si))
          s = dot_row<T, D>(qs[warp], kr + ((size_t)b * S + j) * rs + (size_t)h * D) * scale_log2;
        const float mnew = fmaxf(m, warp_max(s));
        if (mnew == -INFINITY) continue;
        const float alpha = exp2f(m - mnew);
        const float p = exp2f(s - mnew);
        l = l * alpha + warp_sum(p);
#pragma unroll
        for (int u = 0; u < DPL; ++u) acc[u] *= alpha;
        const int nj = (int)min((int64_t)32, t1 - j0);
        for (int jj = 0; jj < nj; ++jj) {
          const float pj = __shfl_sync(kFull, p, jj);
          if (pj != 0.f) {
            const T* vrow = v + ((size_t)b * S + j0 + jj) * rs + (size_t)h * D + lane * DPL;
#pragma unroll
            for (int u = 0; u < DPL; ++u) acc[u] = fmaf(pj, to_f32(vrow[u]), acc[u]);
          }
        }
        m = mnew;
      }
    }
  }
  T* orow = o + tok * rs + (size_t)h * D + lane * DPL;
  const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
  for (int u = 0; u < DPL; ++u) orow[u] = from_f32<T>(acc[u] * inv);
  if (lane == 0) lse[((size_t)b * H + h) * S + i] = l > 0.f ? (m + log2f(l)) * kLn2 : -INFINITY;
}

template <typename T, int D>
__global__ void __launch_bounds__(128)
simt_bwd_dq_kernel(const T* __restrict__ qr, const T* __restrict__ kr, const T* __restrict__ v,
                   const T* __restrict__ d_o, const float* __restrict__ lse,
                   const float* __restrict__ delta, const int32_t* __restrict__ seg,
                   const int32_t* __restrict__ kseg, const int32_t* __restrict__ ktmin,
                   const int32_t* __restrict__ ktmax,
                   T* __restrict__ dq, int64_t S, int H, int64_t n_tiles, float scale,
                   float scale_log2, int causal, double log2_theta, int rotate) {
  constexpr int DPL = D / 32;
  __shared__ float qs[4][D], gs[4][D];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t i = (int64_t)blockIdx.x * 4 + warp;
  const int h = blockIdx.y;
  const int64_t b = blockIdx.z;
  if (i >= S) return;
  const size_t rs = (size_t)H * D;
  const size_t tok = (size_t)b * S + i;
  const size_t hoff = (size_t)h * D;
  for (int d = lane; d < D; d += 32) {
    qs[warp][d] = to_f32(qr[tok * rs + hoff + d]);
    gs[warp][d] = to_f32(d_o[tok * rs + hoff + d]);
  }
  __syncwarp();
  const int32_t si = seg ? seg[tok] : 0;
  const size_t srow = ((size_t)b * H + h) * S + i;
  const float L = lse[srow];
  float acc[DPL];
#pragma unroll
  for (int u = 0; u < DPL; ++u) acc[u] = 0.f;
  if (si >= 0 && L != -INFINITY) {
    const float lse2 = L * kLog2e;
    const float Di = delta[srow];
    const int64_t kend = causal ? i + 1 : S;
    for (int64_t t0 = 0; t0 < kend; t0 += kTile) {
      if (seg && !tile_may_hold(ktmin, ktmax, b * n_tiles + t0 / kTile, si)) continue;
      const int64_t t1 = min(t0 + (int64_t)kTile, kend);
      for (int64_t j0 = t0; j0 < t1; j0 += 32) {
        const int64_t j = j0 + lane;
        float ds = 0.f;
        if (j < t1 && (!seg || kseg[(size_t)b * S + j] == si)) {
          const size_t kro = ((size_t)b * S + j) * rs + hoff;
          const float p = exp2f(dot_row<T, D>(qs[warp], kr + kro) * scale_log2 - lse2);
          const float dp = dot_row<T, D>(gs[warp], v + kro);
          ds = p * (dp - Di);
        }
        const int nj = (int)min((int64_t)32, t1 - j0);
        for (int jj = 0; jj < nj; ++jj) {
          const float dsj = __shfl_sync(kFull, ds, jj);
          if (dsj != 0.f) {
            const T* krow = kr + ((size_t)b * S + j0 + jj) * rs + hoff + lane * DPL;
#pragma unroll
            for (int u = 0; u < DPL; ++u) acc[u] = fmaf(dsj, to_f32(krow[u]), acc[u]);
          }
        }
      }
    }
  }
#pragma unroll
  for (int u = 0; u < DPL; ++u) acc[u] *= scale;
  if (rotate) unrotate_lane<D>(acc, lane, i, log2_theta);
  T* out = dq + tok * rs + hoff + lane * DPL;
#pragma unroll
  for (int u = 0; u < DPL; ++u) out[u] = from_f32<T>(acc[u]);
}

template <typename T, int D>
__global__ void __launch_bounds__(128)
simt_bwd_dkdv_kernel(const T* __restrict__ qr, const T* __restrict__ kr, const T* __restrict__ v,
                     const T* __restrict__ d_o, const float* __restrict__ lse,
                     const float* __restrict__ delta, const int32_t* __restrict__ seg,
                     const int32_t* __restrict__ kseg, const int32_t* __restrict__ tmin,
                     const int32_t* __restrict__ tmax,
                     T* __restrict__ dk, T* __restrict__ dv, int64_t S, int H, int64_t n_tiles,
                     float scale, float scale_log2, int causal, double log2_theta, int rotate) {
  constexpr int DPL = D / 32;
  __shared__ float ks[4][D], vs[4][D];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t j = (int64_t)blockIdx.x * 4 + warp;
  const int h = blockIdx.y;
  const int64_t b = blockIdx.z;
  if (j >= S) return;
  const size_t rs = (size_t)H * D;
  const size_t tok = (size_t)b * S + j;
  const size_t hoff = (size_t)h * D;
  for (int d = lane; d < D; d += 32) {
    ks[warp][d] = to_f32(kr[tok * rs + hoff + d]);
    vs[warp][d] = to_f32(v[tok * rs + hoff + d]);
  }
  __syncwarp();
  const int32_t sj = seg ? kseg[tok] : 0;
  float ak[DPL], av[DPL];
#pragma unroll
  for (int u = 0; u < DPL; ++u) ak[u] = av[u] = 0.f;
  if (sj >= 0) {
    const int64_t istart = causal ? j : 0;
    const size_t lrow = ((size_t)b * H + h) * S;
    for (int64_t t0 = (istart / kTile) * kTile; t0 < S; t0 += kTile) {
      if (seg && !tile_may_hold(tmin, tmax, b * n_tiles + t0 / kTile, sj)) continue;
      const int64_t t1 = min(t0 + (int64_t)kTile, S);
      for (int64_t i0 = t0; i0 < t1; i0 += 32) {
        const int64_t i = i0 + lane;
        float p = 0.f, ds = 0.f;
        if (i < t1 && i >= istart && (!seg || seg[(size_t)b * S + i] == sj)) {
          const float L = lse[lrow + i];
          if (L != -INFINITY) {
            const size_t qro = ((size_t)b * S + i) * rs + hoff;
            p = exp2f(dot_row<T, D>(ks[warp], qr + qro) * scale_log2 - L * kLog2e);
            const float dp = dot_row<T, D>(vs[warp], d_o + qro);
            ds = p * (dp - delta[lrow + i]);
          }
        }
        const int ni = (int)min((int64_t)32, t1 - i0);
        for (int ii = 0; ii < ni; ++ii) {
          const float pj = __shfl_sync(kFull, p, ii);
          const float dsj = __shfl_sync(kFull, ds, ii);
          if (pj != 0.f) {
            const size_t qro = ((size_t)b * S + i0 + ii) * rs + hoff + lane * DPL;
#pragma unroll
            for (int u = 0; u < DPL; ++u) {
              av[u] = fmaf(pj, to_f32(d_o[qro + u]), av[u]);
              ak[u] = fmaf(dsj, to_f32(qr[qro + u]), ak[u]);
            }
          }
        }
      }
    }
  }
#pragma unroll
  for (int u = 0; u < DPL; ++u) ak[u] *= scale;
  if (rotate) unrotate_lane<D>(ak, lane, j, log2_theta);
  T* ok = dk + tok * rs + hoff + lane * DPL;
  T* ov = dv + tok * rs + hoff + lane * DPL;
#pragma unroll
  for (int u = 0; u < DPL; ++u) {
    ok[u] = from_f32<T>(ak[u]);
    ov[u] = from_f32<T>(av[u]);
  }
}

template <typename T, int D>
cudaError_t fwd_impl(const Problem& p, const Workspace& ws, const void* v, void* o, float* lse,
                     cudaStream_t st) {
  dim3 grid((unsigned)((p.S + 3) / 4), (unsigned)p.H, (unsigned)p.B);
  simt_fwd_kernel<T, D><<<grid, 128, 0, st>>>(
      static_cast<const T*>(ws.q_rot), static_cast<const T*>(ws.k_rot), static_cast<const T*>(v),
      static_cast<T*>(o), lse, p.seg, p.kseg, ws.ktile_min, ws.ktile_max, p.S, (int)p.H,
      p.n_tiles, p.scale * kLog2e, p.causal);
  note_launches(1);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t bwd_impl(const Problem& p, const Workspace& ws, const void* v, const float* lse,
                     const void* d_o, void* dq, void* dk, void* dv, cudaStream_t st) {
  dim3 grid((unsigned)((p.S + 3) / 4), (unsigned)p.H, (unsigned)p.B);
  const int rotate = p.theta > 0.0;
  const double l2t = rotate ? log2(p.theta) : 0.0;
  simt_bwd_dq_kernel<T, D><<<grid, 128, 0, st>>>(
      static_cast<const T*>(ws.q_rot), static_cast<const T*>(ws.k_rot), static_cast<const T*>(v),
      static_cast<const T*>(d_o), lse, ws.delta, p.seg, p.kseg, ws.ktile_min, ws.ktile_max,
      static_cast<T*>(dq), p.S, (int)p.H, p.n_tiles, p.scale, p.scale * kLog2e, p.causal, l2t,
      rotate);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  simt_bwd_dkdv_kernel<T, D><<<grid, 128, 0, st>>>(
      static_cast<const T*>(ws.q_rot), static_cast<const T*>(ws.k_rot), static_cast<const T*>(v),
      static_cast<const T*>(d_o), lse, ws.delta, p.seg, p.kseg, ws.tile_min, ws.tile_max,
      static_cast<T*>(dk), static_cast<T*>(dv), p.S, (int)p.H, p.n_tiles, p.scale,
      p.scale * kLog2e, p.causal, l2t, rotate);
  note_launches(2);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_simt_fwd(const Problem& p, const Workspace& ws, const void* v, void* o,
                            float* lse, cudaStream_t st) {
  if (p.B * p.S * p.H == 0) return cudaSuccess;
  if (p.dtype == LWM_DTYPE_BF16)
    return p.D == 64 ? fwd_impl<__nv_bfloat16, 64>(p, ws, v, o, lse, st)
                     : fwd_impl<__nv_bfloat16, 128>(p, ws, v, o, lse, st);
  return p.D == 64 ? fwd_impl<float, 64>(p, ws, v, o, lse, st)
                   : fwd_impl<float, 128>(p, ws, v, o, lse, st);
}

cudaError_t launch_simt_bwd(const Problem& p, const Workspace& ws, const void* v,
                            const float* lse, const void* d_o, void* dq, void* dk, void* dv,
                            cudaStream_t st) {
  if (p.B * p.S * p.H == 0) return cudaSuccess;
  if (p.dtype == LWM_DTYPE_BF16)
    return p.D == 64 ? bwd_impl<__nv_bfloat16, 64>(p, ws, v, lse, d_o, dq, dk, dv, st)
                     : bwd_impl<__nv_bfloat16, 128>(p, ws, v, lse, d_o, dq, dk, dv, st);
  return p.D == 64 ? bwd_impl<float, 64>(p, ws, v, lse, d_o, dq, dk, dv, st)
                   : bwd_impl<float, 128>(p, ws, v, lse, d_o, dq, dk, dv, st);
}

}  // namespace lwm
