// Building blocks of sequence-parallel (ring) attention: the exact merge of
// per-key-block attention results, and fp32 accumulation of per-block
// gradients.
//
// Blockwise RingAttention (LWM research note, "模型架构" and "Infra"; paper
// card, Summary) splits the sequence into blocks held by the devices of a
// ring; each device keeps its query block and sees every key/value block
// once as the blocks travel round the ring.  Attention over the union of key
// blocks is exact when the per-block results are combined by their
// log-sum-exp: with L = ln(e^{L_acc} + e^{L_part}),
//   O <- e^{L_acc - L} O_acc + e^{L_part - L} O_part,   L_acc <- L,
// the same rescaling an online softmax applies inside one kernel.  In the
// backward, each block pair contributes dq, dk, dv computed with the global
// LSE and D = dO . O, and the contributions add up (fp32 here).
#include "common.cuh"
#include "internal.h"

namespace lwm {
namespace {

// One warp per (b, s, h) row; lane l owns elements l, l + 32, ...
template <typename T>
__global__ void __launch_bounds__(256) attn_merge_kernel(float* __restrict__ o_acc,
                                                         float* __restrict__ lse_acc,
                                                         const T* __restrict__ o_part,
                                                         const float* __restrict__ lse_part,
                                                         int64_t n_rows, int64_t S, int H, int D) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= n_rows) return;  // row = (b * S + s) * H + h
  const int64_t h = row % H, tok = row / H;
  const int64_t b = tok / S, s = tok % S;
  const size_t li = ((size_t)b * H + h) * S + s;
  const float la = lse_acc[li], lp = lse_part[li];
  const float m = fmaxf(la, lp);
  float wa = 0.f, wp = 0.f, L = -INFINITY;
  if (m != -INFINITY) {
    const float ea = __expf(la - m), ep = __expf(lp - m);  // 0 for a -inf side
    const float sum = ea + ep;
    wa = ea / sum;
    wp = ep / sum;
    L = m + __logf(sum);
  }
  float* oa = o_acc + (size_t)row * D;
  const T* op = o_part + (size_t)row * D;
  for (int d = lane; d < D; d += 32) oa[d] = wa * oa[d] + wp * to_f32(op[d]);
  if (lane == 0) lse_acc[li] = L;
}

template <typename T>
__global__ void accumulate_kernel(float* __restrict__ acc, const T* __restrict__ x, int64_t n) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x)
    acc[i] += to_f32(x[i]);
}

template <typename T>
__global__ void convert_kernel(const float* __restrict__ x, T* __restrict__ y, int64_t n) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x)
    y[i] = from_f32<T>(x[i]);
}

int elementwise_grid(int64_t n) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t want = (n + 255) / 256, cap = (int64_t)sms * 8;
  return (int)(want < cap ? (want > 0 ? want : 1) : cap);
}

}  // namespace

cudaError_t launch_attn_merge(int64_t B, int64_t S, int64_t H, int64_t D, int dtype, float* o_acc,
                              float* lse_acc, const void* o_part, const float* lse_part,
                              cudaStream_t st) {
  const int64_t rows = B * S * H;
  if (rows == 0) return cudaSuccess;
  const unsigned grid = (unsigned)((rows + 7) / 8);
  if (dtype == LWM_DTYPE_BF16)
    attn_merge_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(
        o_acc, lse_acc, static_cast<const __nv_bfloat16*>(o_part), lse_part, rows, S, (int)H, (int)D);
  else
    attn_merge_kernel<float><<<grid, 256, 0, st>>>(o_acc, lse_acc, static_cast<const float*>(o_part),
                                                   lse_part, rows, S, (int)H, (int)D);
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_accumulate(int64_t n, int dtype, float* acc, const void* x, cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  if (dtype == LWM_DTYPE_BF16)
    accumulate_kernel<<<elementwise_grid(n), 256, 0, st>>>(
        acc, static_cast<const __nv_bfloat16*>(x), n);
  else
    accumulate_kernel<<<elementwise_grid(n), 256, 0, st>>>(acc, static_cast<const float*>(x), n);
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_convert_f32(int64_t n, int dtype, const float* x, void* y, cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  if (dtype == LWM_DTYPE_BF16)
    convert_kernel<<<elementwise_grid(n), 256, 0, st>>>(x, static_cast<__nv_bfloat16*>(y), n);
  else
    convert_kernel<<<elementwise_grid(n), 256, 0, st>>>(x, static_cast<float*>(y), n);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace lwm
