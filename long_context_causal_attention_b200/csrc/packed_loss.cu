// Packed cross-entropy with per-sample re-weighting.
//
// Masked Sequence Packing (LWM research note, "训练方法"; the ablation of
// "评测" shows what naive packing loses): several samples share one row, the
// attention mask keeps them apart, and the loss is re-weighted so that the
// packed batch trains exactly like the samples one by one with padding.
// That reference averages each sample's loss over its own loss tokens and
// then over the samples, so a loss token of a sample with n loss tokens
// weighs 1 / (n * number of samples with a loss token).  A sample is a
// contiguous run of one segment id (what packing produces); ids < 0 are
// padding, targets < 0 tokens without loss.
//
//   run_count_kernel   one CTA per row: the loss-token count n of the run
//                      each token belongs to (a chunk per thread, run
//                      totals stitched across chunk edges by two scans over
//                      the chunk summaries), and the number of samples.
//   ce_kernel          one CTA per token: the row of logits into registers
//                      (16-byte loads, read once from HBM), log-sum-exp, the
//                      weighted loss term and w * (softmax - onehot) (written
//                      once).  HBM-bound: 2 * V * elt bytes per token.
//   loss_sum_kernel    the weighted terms summed in a fixed order.
#include "common.cuh"
#include "internal.h"

namespace lwm {
namespace {

constexpr int kRunThreads = 1024;
constexpr int kCeThreads = 512;
constexpr int kCeVecs = 8;  // 16-byte vectors per thread: V <= 32768 (bf16), 16384 (fp32)

struct ChunkSummary {
  int32_t first_id, last_id;
  int32_t cnt_first, cnt_last;  // loss tokens of the first / last run inside the chunk
  int32_t single;               // the chunk is one run
  int32_t tot_first, tot_last;  // totals of those runs over the whole row
};

__global__ void __launch_bounds__(kRunThreads)
run_count_kernel(const int32_t* __restrict__ seg, const int32_t* __restrict__ targets,
                 int64_t S, int32_t* __restrict__ run_n, int32_t* __restrict__ n_samples) {
  __shared__ ChunkSummary cs[kRunThreads];
  __shared__ int32_t block_samples;
  const int64_t b = blockIdx.x;
  const int tid = threadIdx.x;
  const int64_t chunk = (S + kRunThreads - 1) / kRunThreads;
  const int64_t t0 = (int64_t)tid * chunk, t1 = t0 + chunk < S ? t0 + chunk : S;
  const int32_t* sg = seg ? seg + b * S : nullptr;
  const int32_t* tg = targets + b * S;
  auto id_of = [&](int64_t t) { return sg ? sg[t] : 0; };
  auto loss_tok = [&](int64_t t) { return tg[t] >= 0 && id_of(t) >= 0 ? 1 : 0; };
  if (tid == 0) block_samples = 0;
  ChunkSummary c{};
  if (t0 < t1) {
    c.first_id = id_of(t0);
    c.last_id = id_of(t1 - 1);
    int64_t t = t0;
    while (t < t1 && id_of(t) == c.first_id) c.cnt_first += loss_tok(t++);
    c.single = t == t1;
    t = t1 - 1;
    while (t >= t0 && id_of(t) == c.last_id) c.cnt_last += loss_tok(t--);
  } else {
    c.first_id = c.last_id = INT_MIN;  // empty chunk: joins nothing
    c.single = 0;
  }
  cs[tid] = c;
  __syncthreads();
  if (tid == 0) {
    // left to right: counts of the run open at each chunk's end
    int32_t open_id = INT_MIN, open_cnt = 0;
    for (int i = 0; i < kRunThreads; ++i) {
      ChunkSummary& s = cs[i];
      if (s.first_id == INT_MIN) { open_id = INT_MIN; open_cnt = 0; continue; }
      const int32_t carry = s.first_id == open_id ? open_cnt : 0;
      s.tot_first = carry + s.cnt_first;  // partial: previous chunks' share
      if (s.single) {
        open_cnt = carry + s.cnt_first;
      } else {
        open_cnt = s.cnt_last;
      }
      open_id = s.last_id;
      s.tot_last = open_cnt;  // partial: later chunks add theirs below
    }
    // right to left: complete the totals of runs that cross chunk edges
    int32_t next_id = INT_MIN, next_tot = 0;  // the run starting the next chunk, its total
    for (int i = kRunThreads - 1; i >= 0; --i) {
      ChunkSummary& s = cs[i];
      if (s.first_id == INT_MIN) { next_id = INT_MIN; continue; }
      if (s.last_id == next_id) s.tot_last = next_tot;  // the run continues into the next chunk
      if (s.single) s.tot_first = s.tot_last;
      next_id = s.first_id;
      next_tot = s.tot_first;
    }
  }
  __syncthreads();
  c = cs[tid];
  int32_t samples = 0;
  if (t0 < t1) {
    // walk the chunk: run totals for the first and last run come from the
    // stitched summary, inner runs are counted here
    int64_t t = t0;
    bool first = true;
    while (t < t1) {
      const int32_t id = id_of(t);
      int64_t e = t;
      int32_t cnt = 0;
      while (e < t1 && id_of(e) == id) cnt += loss_tok(e++);
      int32_t tot = cnt;
      if (first) tot = c.tot_first;
      else if (e == t1) tot = c.tot_last;
      // a run starts here unless it continues from the previous chunk
      const bool starts = !(first && t0 > 0 && id_of(t0 - 1) == id);
      if (starts && id >= 0 && tot > 0) ++samples;
      for (int64_t u = t; u < e; ++u) run_n[b * S + u] = id >= 0 ? tot : 0;
      first = false;
      t = e;
    }
  }
  if (samples) atomicAdd(&block_samples, samples);
  __syncthreads();
  if (tid == 0 && block_samples) atomicAdd(n_samples, block_samples);
}

// Block-wide max / sum of one value per thread (kCeThreads threads).
__device__ __forceinline__ float block_max(float v, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  v = red[0];
#pragma unroll
  for (int i = 1; i < kCeThreads / 32; ++i) v = fmaxf(v, red[i]);
  return v;
}

__device__ __forceinline__ float block_sum(float v, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  v = 0.f;
#pragma unroll
  for (int i = 0; i < kCeThreads / 32; ++i) v += red[i];
  return v;
}

// One CTA per token; the row of logits is read once with 16-byte loads into
// registers (NV vectors per thread cover V <= kCeThreads * NV * E, E elements
// per vector), so the log-sum-exp and the gradient need no second read.
template <typename T, int NV>
__global__ void __launch_bounds__(kCeThreads, 2)
ce_kernel(const T* __restrict__ logits, const int32_t* __restrict__ targets,
          const int32_t* __restrict__ run_n, const int32_t* __restrict__ n_samples, int64_t V,
          float* __restrict__ term, T* __restrict__ dlogits) {
  constexpr int E = 16 / sizeof(T);
  __shared__ float red[kCeThreads / 32];
  __shared__ float zy;
  const int64_t tok = blockIdx.x;
  const int tid = threadIdx.x;
  const int32_t y = targets[tok];
  const int32_t n = run_n[tok];
  const int32_t ns = *n_samples;
  // a target outside the vocabulary counts as "no loss" (never read out of range)
  const float w = (y >= 0 && y < V && n > 0 && ns > 0) ? 1.f / ((float)n * (float)ns) : 0.f;
  const int64_t nvec = V / E;  // V is a multiple of E (checked by the caller)
  if (w == 0.f) {  // no loss here: zero gradient row
    if (dlogits) {
      uint4* out = reinterpret_cast<uint4*>(dlogits + tok * V);
      for (int64_t i = tid; i < nvec; i += kCeThreads) out[i] = make_uint4(0, 0, 0, 0);
    }
    if (tid == 0) term[tok] = 0.f;
    return;
  }
  const uint4* row = reinterpret_cast<const uint4*>(logits + tok * V);
  uint4 raw[NV];
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    const int64_t i = tid + (int64_t)k * kCeThreads;
    raw[k] = i < nvec ? __ldg(row + i) : make_uint4(0, 0, 0, 0);
  }
  float mx = -INFINITY;
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    const int64_t i = tid + (int64_t)k * kCeThreads;
    if (i < nvec) {
      const T* e = reinterpret_cast<const T*>(&raw[k]);
#pragma unroll
      for (int u = 0; u < E; ++u) mx = fmaxf(mx, to_f32(e[u]));
    }
  }
  mx = block_max(mx, red);
  float sum = 0.f;
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    const int64_t i = tid + (int64_t)k * kCeThreads;
    if (i < nvec) {
      const T* e = reinterpret_cast<const T*>(&raw[k]);
#pragma unroll
      for (int u = 0; u < E; ++u) {
        const float v = to_f32(e[u]);
        sum += __expf(v - mx);
        if (i * E + u == y) zy = v;
      }
    }
  }
  sum = block_sum(sum, red);  // its barriers also publish zy
  const float lse = mx + __logf(sum);
  if (tid == 0) term[tok] = w * (lse - zy);
  if (dlogits) {
    uint4* out = reinterpret_cast<uint4*>(dlogits + tok * V);
#pragma unroll
    for (int k = 0; k < NV; ++k) {
      const int64_t i = tid + (int64_t)k * kCeThreads;
      if (i < nvec) {
        const T* e = reinterpret_cast<const T*>(&raw[k]);
        uint4 o;
        T* f = reinterpret_cast<T*>(&o);
#pragma unroll
        for (int u = 0; u < E; ++u) {
          const int64_t c = i * E + u;
          f[u] = from_f32<T>(w * (__expf(to_f32(e[u]) - lse) - (c == y ? 1.f : 0.f)));
        }
        out[i] = o;
      }
    }
  }
}

__global__ void __launch_bounds__(1024) loss_sum_kernel(const float* __restrict__ term, int64_t n,
                                                        float* __restrict__ loss) {
  __shared__ double part[1024];
  double acc = 0.0;
  for (int64_t i = threadIdx.x; i < n; i += 1024) acc += term[i];
  part[threadIdx.x] = acc;
  __syncthreads();
  for (int s = 512; s; s >>= 1) {
    if (threadIdx.x < s) part[threadIdx.x] += part[threadIdx.x + s];
    __syncthreads();
  }
  if (threadIdx.x == 0) *loss = (float)part[0];
}

}  // namespace

size_t packed_ce_workspace_bytes(int64_t B, int64_t S) {
  const size_t n = (size_t)B * S;
  return 256 + ((n * 4 + 255) / 256) * 256 * 2;  // sample counter, run_n, terms
}

int64_t packed_ce_max_vocab(int dtype) {
  return (int64_t)kCeThreads * kCeVecs * (dtype == LWM_DTYPE_BF16 ? 8 : 4);
}

cudaError_t launch_packed_ce(int64_t B, int64_t S, int64_t V, int dtype, const void* logits,
                             const int32_t* targets, const int32_t* seg, float* loss,
                             void* dlogits, void* ws, cudaStream_t st) {
  const size_t n = (size_t)B * S;
  char* base = static_cast<char*>(ws);
  int32_t* n_samples = reinterpret_cast<int32_t*>(base);
  int32_t* run_n = reinterpret_cast<int32_t*>(base + 256);
  float* term = reinterpret_cast<float*>(base + 256 + ((n * 4 + 255) / 256) * 256);
  cudaError_t e = cudaMemsetAsync(n_samples, 0, sizeof(int32_t), st);
  if (e != cudaSuccess) return e;
  run_count_kernel<<<(unsigned)B, kRunThreads, 0, st>>>(seg, targets, S, run_n, n_samples);
  if (dtype == LWM_DTYPE_BF16)
    ce_kernel<__nv_bfloat16, kCeVecs><<<(unsigned)n, kCeThreads, 0, st>>>(
        static_cast<const __nv_bfloat16*>(logits), targets, run_n, n_samples, V, term,
        static_cast<__nv_bfloat16*>(dlogits));
  else
    ce_kernel<float, kCeVecs><<<(unsigned)n, kCeThreads, 0, st>>>(
        static_cast<const float*>(logits), targets, run_n, n_samples, V, term,
        static_cast<float*>(dlogits));
  loss_sum_kernel<<<1, 1024, 0, st>>>(term, (int64_t)n, loss);
  note_launches(3);
  return cudaGetLastError();
}

}  // namespace lwm
