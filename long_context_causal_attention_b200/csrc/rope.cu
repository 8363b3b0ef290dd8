// RoPE application (HBM-bound elementwise kernel) and the per-row dot(dO, O).
//
// Rotation as the LWM research note describes it ("模型架构": standard RoPE,
// theta scaled with the context per "训练方法"): pair (x[2t], x[2t+1]) of the
// token at position p turns by p * theta^(-2t/D).
#include "common.cuh"
#include "internal.h"

namespace lwm {
namespace {

// 16-byte vectors: 8 bf16 or 4 fp32 elements (4 or 2 rotary pairs).
template <typename T> struct Vec;
template <> struct Vec<__nv_bfloat16> { static constexpr int N = 8; };
template <> struct Vec<float> { static constexpr int N = 4; };

// One CTA walks tokens with a grid stride.  Thread layout inside a token:
// lane c = tid % (D / N) picks the pair group (fixed for the thread, so its
// frequencies are computed once), hg = tid / (D / N) the head it starts at.
template <typename T>
__global__ void __launch_bounds__(128) rope_kernel(const T* __restrict__ x, T* __restrict__ y,
                                                   int64_t n_tok, int64_t S, int H, int D,
                                                   double log2_theta, int inverse, int64_t pos0) {
  constexpr int N = Vec<T>::N;
  constexpr int P = N / 2;
  const int per_head = D / N;
  const int c = threadIdx.x % per_head;
  const int hg = threadIdx.x / per_head;
  const int heads_per_pass = blockDim.x / per_head;
  if (hg >= heads_per_pass) return;
  double w[P];
#pragma unroll
  for (int u = 0; u < P; ++u) w[u] = rope_freq(c * P + u, D, log2_theta);
  const float sgn = inverse ? -1.0f : 1.0f;
  for (int64_t tok = blockIdx.x; tok < n_tok; tok += gridDim.x) {
    const int64_t pos = pos0 + tok % S;
    float cs[P], sn[P];
#pragma unroll
    for (int u = 0; u < P; ++u) {
      rope_cos_sin_w(pos, w[u], &cs[u], &sn[u]);
      sn[u] *= sgn;
    }
    const size_t base = (size_t)tok * H * D;
    for (int h = hg; h < H; h += heads_per_pass) {
      const size_t off = base + (size_t)h * D + (size_t)c * N;
      uint4 raw = *reinterpret_cast<const uint4*>(x + off);
      T* e = reinterpret_cast<T*>(&raw);
      uint4 outv;
      T* f = reinterpret_cast<T*>(&outv);
#pragma unroll
      for (int u = 0; u < P; ++u) {
        const float a = to_f32(e[2 * u]), b = to_f32(e[2 * u + 1]);
        f[2 * u] = from_f32<T>(a * cs[u] - b * sn[u]);
        f[2 * u + 1] = from_f32<T>(a * sn[u] + b * cs[u]);
      }
      *reinterpret_cast<uint4*>(y + off) = outv;
    }
  }
}

// fp32 operand -> two bf16 planes for the split-precision tensor-core path:
// y = R(p) x when `rotate` (RoPE as rope_kernel computes it), else y = x;
// hi = bf16(y), lo = bf16(y - hi), both rounded to nearest, so hi + lo
// carries y to about 2^-17 relative.  Thread layout as in rope_kernel, four
// fp32 elements (two rotary pairs) per thread and step.
__global__ void __launch_bounds__(128) split_kernel(const float* __restrict__ x,
                                                    __nv_bfloat16* __restrict__ hi,
                                                    __nv_bfloat16* __restrict__ lo, int64_t n_tok,
                                                    int64_t S, int H, int D, double log2_theta,
                                                    int rotate, int64_t pos0) {
  constexpr int N = 4, P = 2;
  const int per_head = D / N;
  const int c = threadIdx.x % per_head;
  const int hg = threadIdx.x / per_head;
  const int heads_per_pass = blockDim.x / per_head;
  if (hg >= heads_per_pass) return;
  double w[P];
#pragma unroll
  for (int u = 0; u < P; ++u) w[u] = rotate ? rope_freq(c * P + u, D, log2_theta) : 0.0;
  for (int64_t tok = blockIdx.x; tok < n_tok; tok += gridDim.x) {
    const int64_t pos = pos0 + tok % S;
    float cs[P] = {1.f, 1.f}, sn[P] = {0.f, 0.f};
    if (rotate) {
#pragma unroll
      for (int u = 0; u < P; ++u) rope_cos_sin_w(pos, w[u], &cs[u], &sn[u]);
    }
    const size_t base = (size_t)tok * H * D;
    for (int h = hg; h < H; h += heads_per_pass) {
      const size_t off = base + (size_t)h * D + (size_t)c * N;
      const float4 v = *reinterpret_cast<const float4*>(x + off);
      const float e[4] = {v.x, v.y, v.z, v.w};
      float y[4];
#pragma unroll
      for (int u = 0; u < P; ++u) {
        y[2 * u] = e[2 * u] * cs[u] - e[2 * u + 1] * sn[u];
        y[2 * u + 1] = e[2 * u] * sn[u] + e[2 * u + 1] * cs[u];
      }
      __nv_bfloat16 h4[4], l4[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        h4[k] = __float2bfloat16_rn(y[k]);
        l4[k] = __float2bfloat16_rn(y[k] - __bfloat162float(h4[k]));
      }
      *reinterpret_cast<uint2*>(hi + off) = *reinterpret_cast<const uint2*>(h4);
      *reinterpret_cast<uint2*>(lo + off) = *reinterpret_cast<const uint2*>(l4);
    }
  }
}

// delta[b, h, i] = sum_d dO[b, i, h, d] * O[b, i, h, d]; one warp per (token, head).
template <typename T>
__global__ void __launch_bounds__(256) delta_kernel(const T* __restrict__ o, const T* __restrict__ d_o,
                                                    float* __restrict__ delta, int64_t n_rows,
                                                    int64_t S, int H, int D) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= n_rows) return;  // row = (b * S + i) * H + h
  const T* a = o + (size_t)row * D;
  const T* g = d_o + (size_t)row * D;
  float acc = 0.f;
  for (int d = lane; d < D; d += 32) acc += to_f32(a[d]) * to_f32(g[d]);
#pragma unroll
  for (int s = 16; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
  if (lane == 0) {
    const int64_t h = row % H, tok = row / H;
    const int64_t b = tok / S, i = tok % S;
    delta[((size_t)b * H + h) * S + i] = acc;
  }
}

// Per (b, h, row) on a row axis padded to whole 128-row tiles:
//   lse2[row] = LSE * log2(e), or +inf when the row has no allowed key or is
//               past the end (so exp2(s - lse2) is exactly 0 there),
//   dpad[row] = dot(dO, O), or 0 past the end.
// One block per batch row and run of `tb` tokens (tb * H rows).  The dot
// products are taken in memory order, a group of D / V lanes per (token,
// head) row with V elements (16 bytes) per lane, so a block streams tb * H
// * D contiguous elements of O and of dO; they go through shared memory so
// that the outputs, laid out head-major, leave tb consecutive rows per head.
template <typename T>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const T* __restrict__ o,
                                                       const T* __restrict__ d_o,
                                                       const float* __restrict__ lse,
                                                       float* __restrict__ lse2,
                                                       float* __restrict__ dpad, int64_t S,
                                                       int64_t S_pad, int H, int D, int tb,
                                                       int64_t n_chunks) {
  extern __shared__ float dots[];  // [tb * H], token-major
  constexpr int V = 16 / sizeof(T);
  const int per_row = D / V;              // lanes per row: 4..32, a power of two
  const int rows_per_warp = 32 / per_row;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int sub = lane % per_row;
  const int64_t b = blockIdx.x / n_chunks;
  const int64_t s0 = (blockIdx.x % n_chunks) * (int64_t)tb;
  const int n_rows = tb * H;
  const size_t base = ((size_t)b * S + (size_t)s0) * H * D;  // first element of token s0
#pragma unroll 4
  for (int r0 = warp * rows_per_warp; r0 < n_rows; r0 += (blockDim.x >> 5) * rows_per_warp) {
    const int rr = r0 + lane / per_row;  // row rr = token s0 + rr / H, head rr % H
    float acc = 0.f;
    if (rr < n_rows && s0 + rr / H < S) {
      const size_t off = base + (size_t)rr * D + (size_t)sub * V;
      const uint4 a = *reinterpret_cast<const uint4*>(o + off);
      const uint4 g = *reinterpret_cast<const uint4*>(d_o + off);
      const T* ea = reinterpret_cast<const T*>(&a);
      const T* eg = reinterpret_cast<const T*>(&g);
#pragma unroll
      for (int e = 0; e < V; ++e) acc += to_f32(ea[e]) * to_f32(eg[e]);
    }
    for (int k = per_row >> 1; k > 0; k >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, k);
    if (rr < n_rows && sub == 0) dots[rr] = acc;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < n_rows; i += blockDim.x) {
    const int h = i / tb, t = i % tb;  // head-major: tb consecutive tokens per head
    const int64_t s = s0 + t;
    if (s >= S_pad) continue;
    float L2 = INFINITY;
    if (s < S) {
      const float L = lse[((size_t)b * H + h) * S + s];
      L2 = L == -INFINITY ? INFINITY : L * 1.4426950408889634f;
    }
    const size_t out = ((size_t)b * H + h) * S_pad + s;
    lse2[out] = L2;
    dpad[out] = s < S ? dots[t * H + h] : 0.f;
  }
}

int grid_for(int64_t n) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t g = (int64_t)sms * 16;
  return (int)(n < g ? (n > 0 ? n : 1) : g);
}

}  // namespace

cudaError_t launch_rope(int64_t B, int64_t S, int64_t H, int64_t D, int dtype, double theta,
                        const void* x, void* y, int inverse, cudaStream_t st, int64_t pos0) {
  const int64_t n_tok = B * S;
  if (n_tok == 0) return cudaSuccess;
  const size_t bytes = (size_t)n_tok * H * D * (dtype == LWM_DTYPE_BF16 ? 2 : 4);
  if (!(theta > 0.0)) {
    if (x == y) return cudaSuccess;
    return cudaMemcpyAsync(y, x, bytes, cudaMemcpyDeviceToDevice, st);
  }
  const double l2t = log2(theta);
  const int grid = grid_for(n_tok);
  if (dtype == LWM_DTYPE_BF16) {
    rope_kernel<__nv_bfloat16><<<grid, 128, 0, st>>>(
        static_cast<const __nv_bfloat16*>(x), static_cast<__nv_bfloat16*>(y), n_tok, S, (int)H,
        (int)D, l2t, inverse, pos0);
  } else {
    rope_kernel<float><<<grid, 128, 0, st>>>(static_cast<const float*>(x), static_cast<float*>(y),
                                             n_tok, S, (int)H, (int)D, l2t, inverse, pos0);
  }
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_split(int64_t B, int64_t S, int64_t H, int64_t D, double theta, const float* x,
                         void* hi, void* lo, cudaStream_t st, int64_t pos0) {
  const int64_t n_tok = B * S;
  if (n_tok == 0) return cudaSuccess;
  const int rotate = theta > 0.0;
  split_kernel<<<grid_for(n_tok), 128, 0, st>>>(x, static_cast<__nv_bfloat16*>(hi),
                                                static_cast<__nv_bfloat16*>(lo), n_tok, S, (int)H,
                                                (int)D, rotate ? log2(theta) : 0.0, rotate, pos0);
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_delta(const Problem& p, const void* o, const void* d_o, float* delta,
                         cudaStream_t st) {
  const int64_t rows = p.B * p.S * p.H;
  if (rows == 0) return cudaSuccess;
  const int64_t grid = (rows + 7) / 8;
  if (p.dtype == LWM_DTYPE_BF16) {
    delta_kernel<__nv_bfloat16><<<(unsigned)grid, 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(d_o), delta, rows,
        p.S, (int)p.H, (int)p.D);
  } else {
    delta_kernel<float><<<(unsigned)grid, 256, 0, st>>>(static_cast<const float*>(o),
                                                       static_cast<const float*>(d_o), delta, rows,
                                                       p.S, (int)p.H, (int)p.D);
  }
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_bwd_prep(const Problem& p, const void* o, const void* d_o, const float* lse,
                            const Workspace& ws, cudaStream_t st) {
  const int64_t s_pad = p.n_tiles * kTile;
  if (p.B * p.H * s_pad == 0) return cudaSuccess;
  // tokens per block: about 256 (token, head) rows, a multiple of 8 tokens
  // where H allows (whole 32-byte sectors of the head-major outputs)
  int tb = (int)(256 / p.H);
  if (tb >= 8) tb &= ~7;
  if (tb < 1) tb = 1;
  const int64_t n_chunks = (s_pad + tb - 1) / tb;
  const int64_t grid = p.B * n_chunks;
  const size_t smem = (size_t)tb * p.H * sizeof(float);
  if (smem > 48 * 1024) return cudaErrorInvalidValue;  // H above 12288
  if (p.dtype == LWM_DTYPE_BF16)
    bwd_prep_kernel<__nv_bfloat16><<<(unsigned)grid, 256, smem, st>>>(
        static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(d_o), lse,
        ws.lse2_pad, ws.delta_pad, p.S, s_pad, (int)p.H, (int)p.D, tb, n_chunks);
  else
    bwd_prep_kernel<float><<<(unsigned)grid, 256, smem, st>>>(
        static_cast<const float*>(o), static_cast<const float*>(d_o), lse, ws.lse2_pad,
        ws.delta_pad, p.S, s_pad, (int)p.H, (int)p.D, tb, n_chunks);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace lwm
