// CUDA-core (SIMT, fp32 arithmetic) attention kernels.
//
// These serve the fp32 data type, where the answer must agree with the exact
// result to 1e-4 and tensor-core tf32 cannot, and head_dim 64.  A CTA of 256
// threads owns a block of 64 query rows (forward, dQ) or 64 key rows (dK/dV)
// and sweeps the 64-row blocks of the other side through shared memory, held
// there as fp32 whatever the input type.  Every product is a register-tiled
// contraction out of shared memory with 16-byte loads:
//   score tiles (64 x 64)     thread (ty, tx) holds rows 4ty..4ty+3 and
//                             columns tx, tx+16, tx+32, tx+48
//   accumulators (64 x D)     rows 4ty..4ty+3, columns 64c + 4tx .. +3
// with ty = thread / 16 and tx = thread % 16.  The 16 threads of a row group
// form one half-warp, so a row max or sum is four shuffles.  Rows of the
// 64 x D tiles are padded to D + 4 floats and score tiles to 68, which keeps
// every shared-memory access at the minimum number of wavefronts.
//
// Math (LWM research note, "模型架构": exact blockwise attention with online
// softmax; "训练方法": packing mask; backward recomputes P from LSE as in the
// FlashAttention entry of the paper card's references):
//   forward   m, l running max / sum in log2 units, O = sum p v / l,
//             LSE = (m + log2 l) ln 2
//   dQ        dS_ij = P_ij (dO_i.v_j - D_i),  dq~_i = scale sum_j dS_ij k~_j
//   dK/dV     dv_j = sum_i P_ij dO_i,  dk~_j = scale sum_i dS_ij q~_i
// Gradients are turned back from the rotated frame with R(p)^T in the
// epilogue (no separate pass, no atomics).  Whole 64 x 64 blocks are skipped
// when the 128-token tile bounds of the segment prepass show that no pair in
// them can share a segment.
#include <climits>
#include <cmath>

#include "common.cuh"
#include "internal.h"

namespace lwm {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr unsigned kFull = 0xffffffffu;
constexpr int kBlk = 64;            // rows per block on either side
constexpr int kThreads = 256;
constexpr int kPld = kBlk + 4;      // row stride of a 64 x 64 score tile, floats
constexpr int kSubPerTile = kTile / kBlk;

template <int D> __host__ __device__ constexpr int tile_ld() { return D + 4; }
template <int D> __host__ __device__ constexpr int tile_floats() { return kBlk * tile_ld<D>(); }

__device__ __forceinline__ float group_max(float x) {  // over the 16 lanes of a half-warp
#pragma unroll
  for (int s = 8; s > 0; s >>= 1) x = fmaxf(x, __shfl_xor_sync(kFull, x, s));
  return x;
}
__device__ __forceinline__ float group_sum(float x) {
#pragma unroll
  for (int s = 8; s > 0; s >>= 1) x += __shfl_xor_sync(kFull, x, s);
  return x;
}

__device__ __forceinline__ float comp(const float4& v, int i) {
  return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

// Can a pair of 128-token tiles (query tile qt, key tile kt, both already
// offset by the row's tile base) hold an allowed pair?  Bounds as the segment
// prepass writes them: min is -1 for a tile with padding, max is -1 for a
// tile without a valid token.
__device__ __forceinline__ bool tiles_meet(const int32_t* tmin, const int32_t* tmax,
                                           const int32_t* ktmin, const int32_t* ktmax,
                                           int64_t qt, int64_t kt) {
  const int32_t a0 = tmin[qt], a1 = tmax[qt], b0 = ktmin[kt], b1 = ktmax[kt];
  return a1 >= 0 && b1 >= 0 && a0 <= b1 && b0 <= a1;
}

// Rows [r0, r0 + 64) of one head -> dst[64][D + 4] as fp32, rows at or past S
// as zeros.  src points at (b, token 0, h, 0); row_stride = H * D elements.
template <typename T, int D>
__device__ __forceinline__ void load_tile(float* __restrict__ dst, const T* __restrict__ src,
                                          size_t row_stride, int64_t r0, int64_t S) {
  constexpr int kEpc = 16 / (int)sizeof(T);  // elements per 16-byte chunk
  constexpr int kCpr = D / kEpc;             // chunks per row
  constexpr int LD = tile_ld<D>();
  static_assert((kBlk * kCpr) % kThreads == 0, "tile chunks must divide evenly");
#pragma unroll
  for (int it = 0; it < kBlk * kCpr / kThreads; ++it) {
    const int f = threadIdx.x + it * kThreads;
    const int r = f / kCpr, c = f % kCpr;
    float* d = dst + r * LD + c * kEpc;
    if (r0 + r < S) {
      const uint4 raw =
          __ldg(reinterpret_cast<const uint4*>(src + (size_t)(r0 + r) * row_stride) + c);
      const T* e = reinterpret_cast<const T*>(&raw);
#pragma unroll
      for (int u = 0; u < kEpc; u += 4)
        *reinterpret_cast<float4*>(d + u) =
            make_float4(to_f32(e[u]), to_f32(e[u + 1]), to_f32(e[u + 2]), to_f32(e[u + 3]));
    } else {
#pragma unroll
      for (int u = 0; u < kEpc; u += 4)
        *reinterpret_cast<float4*>(d + u) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
}

// s[r][c] += <A row 4ty+r, B row tx+16c> over D columns (A, B: [64][D + 4]).
template <int D>
__device__ __forceinline__ void rows_dot_rows(const float* __restrict__ A,
                                              const float* __restrict__ B, int ty, int tx,
                                              float s[4][4]) {
  constexpr int LD = tile_ld<D>();
  const float* a = A + 4 * ty * LD;
  const float* b = B + tx * LD;
#pragma unroll 4
  for (int d = 0; d < D; d += 4) {
    float4 x[4], y[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) x[r] = *reinterpret_cast<const float4*>(a + r * LD + d);
#pragma unroll
    for (int c = 0; c < 4; ++c) y[c] = *reinterpret_cast<const float4*>(b + 16 * c * LD + d);
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        s[r][c] = fmaf(x[r].x, y[c].x, s[r][c]);
        s[r][c] = fmaf(x[r].y, y[c].y, s[r][c]);
        s[r][c] = fmaf(x[r].z, y[c].z, s[r][c]);
        s[r][c] = fmaf(x[r].w, y[c].w, s[r][c]);
      }
  }
}

// acc[r][4c+e] += sum_k P[4ty+r][k] B[k][64c + 4tx + e]  (P: [64][68], B: [64][D + 4]).
template <int D>
__device__ __forceinline__ void rows_times_tile(const float* __restrict__ P,
                                                const float* __restrict__ B, int ty, int tx,
                                                float acc[4][D / 16]) {
  constexpr int LD = tile_ld<D>(), NC = D / 64;
  const float* p = P + 4 * ty * kPld;
  const float* b = B + 4 * tx;
#pragma unroll 2
  for (int k = 0; k < kBlk; k += 4) {
    float4 x[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) x[r] = *reinterpret_cast<const float4*>(p + r * kPld + k);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        const float4 y = *reinterpret_cast<const float4*>(b + (k + kk) * LD + 64 * c);
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const float xr = comp(x[r], kk);
          acc[r][4 * c + 0] = fmaf(xr, y.x, acc[r][4 * c + 0]);
          acc[r][4 * c + 1] = fmaf(xr, y.y, acc[r][4 * c + 1]);
          acc[r][4 * c + 2] = fmaf(xr, y.z, acc[r][4 * c + 2]);
          acc[r][4 * c + 3] = fmaf(xr, y.w, acc[r][4 * c + 3]);
        }
      }
  }
}

// acc[r][4c+e] += sum_q P[q][4ty+r] B[q][64c + 4tx + e]  (the left operand transposed).
template <int D>
__device__ __forceinline__ void cols_times_tile(const float* __restrict__ P,
                                                const float* __restrict__ B, int ty, int tx,
                                                float acc[4][D / 16]) {
  constexpr int LD = tile_ld<D>(), NC = D / 64;
  const float* p = P + 4 * ty;
  const float* b = B + 4 * tx;
#pragma unroll 4
  for (int q = 0; q < kBlk; ++q) {
    const float4 x = *reinterpret_cast<const float4*>(p + q * kPld);
#pragma unroll
    for (int c = 0; c < NC; ++c) {
      const float4 y = *reinterpret_cast<const float4*>(b + q * LD + 64 * c);
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const float xr = comp(x, r);
        acc[r][4 * c + 0] = fmaf(xr, y.x, acc[r][4 * c + 0]);
        acc[r][4 * c + 1] = fmaf(xr, y.y, acc[r][4 * c + 1]);
        acc[r][4 * c + 2] = fmaf(xr, y.z, acc[r][4 * c + 2]);
        acc[r][4 * c + 3] = fmaf(xr, y.w, acc[r][4 * c + 3]);
      }
    }
  }
}

template <typename T> __device__ __forceinline__ void store4(T* dst, const float* x);
template <> __device__ __forceinline__ void store4<float>(float* dst, const float* x) {
  *reinterpret_cast<float4*>(dst) = make_float4(x[0], x[1], x[2], x[3]);
}
template <> __device__ __forceinline__ void store4<__nv_bfloat16>(__nv_bfloat16* dst,
                                                                  const float* x) {
  __nv_bfloat162 lo = __floats2bfloat162_rn(x[0], x[1]);
  __nv_bfloat162 hi = __floats2bfloat162_rn(x[2], x[3]);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t*>(&lo);
  u.y = *reinterpret_cast<uint32_t*>(&hi);
  *reinterpret_cast<uint2*>(dst) = u;
}

// R(pos)^T on four consecutive dims d0..d0+3 (two rotation pairs), in place.
template <int D>
__device__ __forceinline__ void unrotate4(float* x, int d0, int64_t pos, double log2_theta) {
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    float c, s;
    rope_cos_sin_w(pos, rope_freq(d0 / 2 + u, D, log2_theta), &c, &s);
    const float a = x[2 * u], b = x[2 * u + 1];
    x[2 * u] = a * c + b * s;
    x[2 * u + 1] = b * c - a * s;
  }
}

// First 64-key block a query block needs (segment bounds, else 0).
__device__ __forceinline__ int64_t first_key_block(const int32_t* seg, const int32_t* q_lo,
                                                   int64_t b, int64_t n_tiles, int64_t qt) {
  return seg ? (int64_t)q_lo[b * n_tiles + qt] * kSubPerTile : 0;
}

// ---------------------------------------------------------------------------
// forward: one CTA per (64 query rows, head, batch row)
// ---------------------------------------------------------------------------
template <int D> constexpr size_t fwd_smem_bytes() {
  return (size_t)(2 * tile_floats<D>() + kBlk * kPld) * sizeof(float) + kBlk * sizeof(int32_t);
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads, 2)
simt_fwd_kernel(const T* __restrict__ qr, const T* __restrict__ kr, const T* __restrict__ v,
                T* __restrict__ o, float* __restrict__ lse, const int32_t* __restrict__ seg,
                const int32_t* __restrict__ kseg, const int32_t* __restrict__ tmin,
                const int32_t* __restrict__ tmax, const int32_t* __restrict__ ktmin,
                const int32_t* __restrict__ ktmax, const int32_t* __restrict__ q_lo, int64_t S,
                int H, int64_t n_tiles, float scale_log2, int causal) {
  constexpr int NA = D / 16, NC = D / 64;
  extern __shared__ float4 smem_f4[];
  float* Qs = reinterpret_cast<float*>(smem_f4);
  float* KVs = Qs + tile_floats<D>();
  float* Ps = KVs + tile_floats<D>();
  int32_t* kseg_s = reinterpret_cast<int32_t*>(Ps + kBlk * kPld);

  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  const int64_t nqb = (S + kBlk - 1) / kBlk;
  const int64_t qb = nqb - 1 - (int64_t)blockIdx.x;  // longest causal rows first
  const int h = blockIdx.y;
  const int64_t b = blockIdx.z;
  const int64_t i0 = qb * kBlk;
  const size_t rs = (size_t)H * D;
  const size_t head = (size_t)b * S * rs + (size_t)h * D;

  load_tile<T, D>(Qs, qr + head, rs, i0, S);
  int32_t si[4];
  float m[4], l[4], acc[4][NA];
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int64_t i = i0 + 4 * ty + r;
    si[r] = i < S ? (seg ? seg[b * S + i] : 0) : -1;
    m[r] = -INFINITY;
    l[r] = 0.f;
#pragma unroll
    for (int a = 0; a < NA; ++a) acc[r][a] = 0.f;
  }

  const int64_t qt = i0 / kTile;
  const int64_t kend = causal ? min(S, i0 + kBlk) : S;
  const int64_t nkb = (kend + kBlk - 1) / kBlk;
  for (int64_t kb = first_key_block(seg, q_lo, b, n_tiles, qt); kb < nkb; ++kb) {
    const int64_t j0 = kb * kBlk;
    if (seg && !tiles_meet(tmin, tmax, ktmin, ktmax, b * n_tiles + qt, b * n_tiles + j0 / kTile))
      continue;
    __syncthreads();  // the previous block's P.V reads are done
    load_tile<T, D>(KVs, kr + head, rs, j0, S);
    if (tid < kBlk) kseg_s[tid] = j0 + tid < S ? (seg ? kseg[b * S + j0 + tid] : 0) : INT_MIN;
    __syncthreads();

    float s[4][4];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int c = 0; c < 4; ++c) s[r][c] = 0.f;
    rows_dot_rows<D>(Qs, KVs, ty, tx, s);

#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int64_t i = i0 + 4 * ty + r;
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int jl = tx + 16 * c;
        const bool ok = si[r] >= 0 && kseg_s[jl] == si[r] && (!causal || j0 + jl <= i);
        s[r][c] = ok ? s[r][c] * scale_log2 : -INFINITY;
        mx = fmaxf(mx, s[r][c]);
      }
      const float mnew = fmaxf(m[r], group_max(mx));
      const float mu = mnew == -INFINITY ? 0.f : mnew;
      const float alpha = exp2f(m[r] - mu);
      m[r] = mnew;
      float psum = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const float p = exp2f(s[r][c] - mu);
        Ps[(4 * ty + r) * kPld + tx + 16 * c] = p;
        psum += p;
      }
      l[r] = l[r] * alpha + psum;
#pragma unroll
      for (int a = 0; a < NA; ++a) acc[r][a] *= alpha;
    }
    __syncthreads();  // every read of K is done: V takes its place
    load_tile<T, D>(KVs, v + head, rs, j0, S);
    __syncthreads();
    rows_times_tile<D>(Ps, KVs, ty, tx, acc);
  }

#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const float lt = group_sum(l[r]);
    const int64_t i = i0 + 4 * ty + r;
    if (i < S) {
      const float inv = lt > 0.f ? 1.f / lt : 0.f;
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        float x[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) x[e] = acc[r][4 * c + e] * inv;
        store4<T>(o + head + (size_t)i * rs + 64 * c + 4 * tx, x);
      }
      if (tx == 0)
        lse[((size_t)b * H + h) * S + i] = lt > 0.f ? (m[r] + log2f(lt)) * kLn2 : -INFINITY;
    }
  }
}

// ---------------------------------------------------------------------------
// backward dK/dV: one CTA per (64 key rows, head, batch row)
// ---------------------------------------------------------------------------
template <int D> constexpr size_t dkdv_smem_bytes() {
  return (size_t)(4 * tile_floats<D>() + 2 * kBlk * kPld) * sizeof(float) +
         3 * kBlk * sizeof(float);
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads, 1)
simt_bwd_dkdv_kernel(const T* __restrict__ qr, const T* __restrict__ kr, const T* __restrict__ v,
                     const T* __restrict__ d_o, const float* __restrict__ lse,
                     const float* __restrict__ delta, const int32_t* __restrict__ seg,
                     const int32_t* __restrict__ kseg, const int32_t* __restrict__ tmin,
                     const int32_t* __restrict__ tmax, const int32_t* __restrict__ ktmin,
                     const int32_t* __restrict__ ktmax, const int32_t* __restrict__ k_hi,
                     T* __restrict__ dk, T* __restrict__ dv, int64_t S, int H, int64_t n_tiles,
                     float scale, float scale_log2, int causal, double log2_theta, int rotate) {
  constexpr int NA = D / 16, NC = D / 64;
  extern __shared__ float4 smem_f4[];
  float* Ks = reinterpret_cast<float*>(smem_f4);
  float* Vs = Ks + tile_floats<D>();
  float* Qs = Vs + tile_floats<D>();
  float* Gs = Qs + tile_floats<D>();  // dO
  float* Ps = Gs + tile_floats<D>();
  float* dSs = Ps + kBlk * kPld;
  float* lse2_s = dSs + kBlk * kPld;
  float* delta_s = lse2_s + kBlk;
  int32_t* qseg_s = reinterpret_cast<int32_t*>(delta_s + kBlk);

  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  const int64_t kb = blockIdx.x;  // causal: the first key blocks see the most queries
  const int h = blockIdx.y;
  const int64_t b = blockIdx.z;
  const int64_t j0 = kb * kBlk;
  const size_t rs = (size_t)H * D;
  const size_t head = (size_t)b * S * rs + (size_t)h * D;
  const size_t lrow = ((size_t)b * H + h) * S;

  load_tile<T, D>(Ks, kr + head, rs, j0, S);
  load_tile<T, D>(Vs, v + head, rs, j0, S);
  int32_t sj[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const int64_t j = j0 + tx + 16 * c;
    sj[c] = j < S ? (seg ? kseg[b * S + j] : 0) : INT_MIN;
  }
  float ak[4][NA], av[4][NA];
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int a = 0; a < NA; ++a) ak[r][a] = av[r][a] = 0.f;

  const int64_t kt = j0 / kTile;
  const int64_t nqb = (S + kBlk - 1) / kBlk;
  int64_t qb_end = nqb - 1;
  if (seg) qb_end = min(qb_end, (int64_t)k_hi[b * n_tiles + kt] * kSubPerTile + kSubPerTile - 1);
  for (int64_t qb = causal ? kb : 0; qb <= qb_end; ++qb) {
    const int64_t i0 = qb * kBlk;
    if (seg && !tiles_meet(tmin, tmax, ktmin, ktmax, b * n_tiles + i0 / kTile, b * n_tiles + kt))
      continue;
    __syncthreads();  // the previous block's dV/dK reads are done
    load_tile<T, D>(Qs, qr + head, rs, i0, S);
    load_tile<T, D>(Gs, d_o + head, rs, i0, S);
    if (tid < kBlk) {
      const int64_t i = i0 + tid;
      const float L = i < S ? lse[lrow + i] : -INFINITY;
      const bool live = L != -INFINITY;
      qseg_s[tid] = live ? (seg ? seg[b * S + i] : 0) : -1;
      lse2_s[tid] = live ? L * kLog2e : 0.f;
      delta_s[tid] = live ? delta[lrow + i] : 0.f;
    }
    __syncthreads();

    float s[4][4], dp[4][4];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int c = 0; c < 4; ++c) s[r][c] = dp[r][c] = 0.f;
    rows_dot_rows<D>(Qs, Ks, ty, tx, s);   // rows: queries, columns: keys
    rows_dot_rows<D>(Gs, Vs, ty, tx, dp);
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int il = 4 * ty + r;
      const int32_t qs = qseg_s[il];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int jl = tx + 16 * c;
        const bool ok = qs >= 0 && qs == sj[c] && (!causal || j0 + jl <= i0 + il);
        const float p = ok ? exp2f(s[r][c] * scale_log2 - lse2_s[il]) : 0.f;
        Ps[il * kPld + jl] = p;
        dSs[il * kPld + jl] = p * (dp[r][c] - delta_s[il]);
      }
    }
    __syncthreads();
    cols_times_tile<D>(Ps, Gs, ty, tx, av);   // rows: keys 4ty..
    cols_times_tile<D>(dSs, Qs, ty, tx, ak);
  }

#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int64_t j = j0 + 4 * ty + r;
    if (j >= S) continue;
#pragma unroll
    for (int c = 0; c < NC; ++c) {
      float xk[4], xv[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        xk[e] = ak[r][4 * c + e] * scale;
        xv[e] = av[r][4 * c + e];
      }
      if (rotate) unrotate4<D>(xk, 64 * c + 4 * tx, j, log2_theta);
      store4<T>(dk + head + (size_t)j * rs + 64 * c + 4 * tx, xk);
      store4<T>(dv + head + (size_t)j * rs + 64 * c + 4 * tx, xv);
    }
  }
}

// ---------------------------------------------------------------------------
// backward dQ: one CTA per (64 query rows, head, batch row)
// ---------------------------------------------------------------------------
template <int D> constexpr size_t dq_smem_bytes() {
  return (size_t)(4 * tile_floats<D>() + kBlk * kPld) * sizeof(float) + kBlk * sizeof(int32_t);
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads, 1)
simt_bwd_dq_kernel(const T* __restrict__ qr, const T* __restrict__ kr, const T* __restrict__ v,
                   const T* __restrict__ d_o, const float* __restrict__ lse,
                   const float* __restrict__ delta, const int32_t* __restrict__ seg,
                   const int32_t* __restrict__ kseg, const int32_t* __restrict__ tmin,
                   const int32_t* __restrict__ tmax, const int32_t* __restrict__ ktmin,
                   const int32_t* __restrict__ ktmax, const int32_t* __restrict__ q_lo,
                   T* __restrict__ dq, int64_t S, int H, int64_t n_tiles, float scale,
                   float scale_log2, int causal, double log2_theta, int rotate) {
  constexpr int NA = D / 16, NC = D / 64;
  extern __shared__ float4 smem_f4[];
  float* Qs = reinterpret_cast<float*>(smem_f4);
  float* Gs = Qs + tile_floats<D>();  // dO
  float* Ks = Gs + tile_floats<D>();
  float* Vs = Ks + tile_floats<D>();
  float* dSs = Vs + tile_floats<D>();
  int32_t* kseg_s = reinterpret_cast<int32_t*>(dSs + kBlk * kPld);

  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  const int64_t nqb = (S + kBlk - 1) / kBlk;
  const int64_t qb = nqb - 1 - (int64_t)blockIdx.x;
  const int h = blockIdx.y;
  const int64_t b = blockIdx.z;
  const int64_t i0 = qb * kBlk;
  const size_t rs = (size_t)H * D;
  const size_t head = (size_t)b * S * rs + (size_t)h * D;
  const size_t lrow = ((size_t)b * H + h) * S;

  load_tile<T, D>(Qs, qr + head, rs, i0, S);
  load_tile<T, D>(Gs, d_o + head, rs, i0, S);
  int32_t si[4];
  float lse2[4], dl[4], acc[4][NA];
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int64_t i = i0 + 4 * ty + r;
    const float L = i < S ? lse[lrow + i] : -INFINITY;
    const bool live = L != -INFINITY;
    si[r] = live ? (seg ? seg[b * S + i] : 0) : -1;
    lse2[r] = live ? L * kLog2e : 0.f;
    dl[r] = live ? delta[lrow + i] : 0.f;
#pragma unroll
    for (int a = 0; a < NA; ++a) acc[r][a] = 0.f;
  }

  const int64_t qt = i0 / kTile;
  const int64_t kend = causal ? min(S, i0 + kBlk) : S;
  const int64_t nkb = (kend + kBlk - 1) / kBlk;
  for (int64_t kb = first_key_block(seg, q_lo, b, n_tiles, qt); kb < nkb; ++kb) {
    const int64_t j0 = kb * kBlk;
    if (seg && !tiles_meet(tmin, tmax, ktmin, ktmax, b * n_tiles + qt, b * n_tiles + j0 / kTile))
      continue;
    __syncthreads();  // the previous block's dS.K reads are done
    load_tile<T, D>(Ks, kr + head, rs, j0, S);
    load_tile<T, D>(Vs, v + head, rs, j0, S);
    if (tid < kBlk) kseg_s[tid] = j0 + tid < S ? (seg ? kseg[b * S + j0 + tid] : 0) : INT_MIN;
    __syncthreads();

    float s[4][4], dp[4][4];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int c = 0; c < 4; ++c) s[r][c] = dp[r][c] = 0.f;
    rows_dot_rows<D>(Qs, Ks, ty, tx, s);
    rows_dot_rows<D>(Gs, Vs, ty, tx, dp);
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int il = 4 * ty + r;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int jl = tx + 16 * c;
        const bool ok = si[r] >= 0 && kseg_s[jl] == si[r] && (!causal || j0 + jl <= i0 + il);
        const float p = ok ? exp2f(s[r][c] * scale_log2 - lse2[r]) : 0.f;
        dSs[il * kPld + jl] = p * (dp[r][c] - dl[r]);
      }
    }
    __syncthreads();
    rows_times_tile<D>(dSs, Ks, ty, tx, acc);
  }

#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int64_t i = i0 + 4 * ty + r;
    if (i >= S) continue;
#pragma unroll
    for (int c = 0; c < NC; ++c) {
      float x[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) x[e] = acc[r][4 * c + e] * scale;
      if (rotate) unrotate4<D>(x, 64 * c + 4 * tx, i, log2_theta);
      store4<T>(dq + head + (size_t)i * rs + 64 * c + 4 * tx, x);
    }
  }
}

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------
template <typename T, int D>
cudaError_t fwd_impl(const Problem& p, const Workspace& ws, const void* v, void* o, float* lse,
                     cudaStream_t st) {
  constexpr size_t smem = fwd_smem_bytes<D>();
  cudaError_t e = cudaFuncSetAttribute(simt_fwd_kernel<T, D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)((p.S + kBlk - 1) / kBlk), (unsigned)p.H, (unsigned)p.B);
  simt_fwd_kernel<T, D><<<grid, kThreads, smem, st>>>(
      static_cast<const T*>(ws.q_rot), static_cast<const T*>(ws.k_rot), static_cast<const T*>(v),
      static_cast<T*>(o), lse, p.seg, p.kseg, ws.tile_min, ws.tile_max, ws.ktile_min,
      ws.ktile_max, ws.q_lo, p.S, (int)p.H, p.n_tiles, p.scale * kLog2e, p.causal);
  note_launches(1);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t dkdv_impl(const Problem& p, const Workspace& ws, const void* v, const float* lse,
                      const void* d_o, void* dk, void* dv, cudaStream_t st) {
  constexpr size_t smem = dkdv_smem_bytes<D>();
  cudaError_t e = cudaFuncSetAttribute(simt_bwd_dkdv_kernel<T, D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int rotate = p.theta > 0.0;
  dim3 grid((unsigned)((p.S + kBlk - 1) / kBlk), (unsigned)p.H, (unsigned)p.B);
  simt_bwd_dkdv_kernel<T, D><<<grid, kThreads, smem, st>>>(
      static_cast<const T*>(ws.q_rot), static_cast<const T*>(ws.k_rot), static_cast<const T*>(v),
      static_cast<const T*>(d_o), lse, ws.delta, p.seg, p.kseg, ws.tile_min, ws.tile_max,
      ws.ktile_min, ws.ktile_max, ws.k_hi, static_cast<T*>(dk), static_cast<T*>(dv), p.S,
      (int)p.H, p.n_tiles, p.scale, p.scale * kLog2e, p.causal, rotate ? log2(p.theta) : 0.0,
      rotate);
  note_launches(1);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t dq_impl(const Problem& p, const Workspace& ws, const void* v, const float* lse,
                    const void* d_o, void* dq, cudaStream_t st) {
  constexpr size_t smem = dq_smem_bytes<D>();
  cudaError_t e = cudaFuncSetAttribute(simt_bwd_dq_kernel<T, D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int rotate = p.theta > 0.0;
  dim3 grid((unsigned)((p.S + kBlk - 1) / kBlk), (unsigned)p.H, (unsigned)p.B);
  simt_bwd_dq_kernel<T, D><<<grid, kThreads, smem, st>>>(
      static_cast<const T*>(ws.q_rot), static_cast<const T*>(ws.k_rot), static_cast<const T*>(v),
      static_cast<const T*>(d_o), lse, ws.delta, p.seg, p.kseg, ws.tile_min, ws.tile_max,
      ws.ktile_min, ws.ktile_max, ws.q_lo, static_cast<T*>(dq), p.S, (int)p.H, p.n_tiles,
      p.scale, p.scale * kLog2e, p.causal, rotate ? log2(p.theta) : 0.0, rotate);
  note_launches(1);
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

cudaError_t launch_simt_bwd_dkdv(const Problem& p, const Workspace& ws, const void* v,
                                 const float* lse, const void* d_o, void* dk, void* dv,
                                 cudaStream_t st) {
  if (p.B * p.S * p.H == 0) return cudaSuccess;
  if (p.dtype == LWM_DTYPE_BF16)
    return p.D == 64 ? dkdv_impl<__nv_bfloat16, 64>(p, ws, v, lse, d_o, dk, dv, st)
                     : dkdv_impl<__nv_bfloat16, 128>(p, ws, v, lse, d_o, dk, dv, st);
  return p.D == 64 ? dkdv_impl<float, 64>(p, ws, v, lse, d_o, dk, dv, st)
                   : dkdv_impl<float, 128>(p, ws, v, lse, d_o, dk, dv, st);
}

cudaError_t launch_simt_bwd_dq(const Problem& p, const Workspace& ws, const void* v,
                               const float* lse, const void* d_o, void* dq, cudaStream_t st) {
  if (p.B * p.S * p.H == 0) return cudaSuccess;
  if (p.dtype == LWM_DTYPE_BF16)
    return p.D == 64 ? dq_impl<__nv_bfloat16, 64>(p, ws, v, lse, d_o, dq, st)
                     : dq_impl<__nv_bfloat16, 128>(p, ws, v, lse, d_o, dq, st);
  return p.D == 64 ? dq_impl<float, 64>(p, ws, v, lse, d_o, dq, st)
                   : dq_impl<float, 128>(p, ws, v, lse, d_o, dq, st);
}

}  // namespace lwm
