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
// padding, targets < 0 or >= V tokens without loss.
//
//   run_count_kernel   one CTA per row: the loss-token count n of the run
//                      each token belongs to (a chunk per thread, run
//                      totals stitched across chunk edges by two scans over
//                      the chunk summaries), and the number of samples.
//   ce_kernel          persistent, one CTA per SM, rows round-robin.  A
//                      producer warp streams the rows that carry a loss into
//                      a ring of shared-memory stages with bulk async copies
//                      (several rows in flight per SM); 16 consumer warps
//                      move a row into registers, free its stage at once and
//                      compute the log-sum-exp, the weighted loss term and
//                      w * (softmax - onehot) (written once).  Rows without a
//                      loss pass through the ring without data and get a zero
//                      gradient.  HBM-bound: 2 * V * elt bytes per token.
//   loss_sum_kernel    the weighted terms summed in a fixed order.
#include <algorithm>
#include <type_traits>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace lwm {
namespace {

constexpr int kRunThreads = 256;  // chunks per row: short serial stitching scans
constexpr int kCeConsumerWarps = 16;
constexpr int kCeConsumers = kCeConsumerWarps * 32;  // threads that hold a row
constexpr int kCeThreads = kCeConsumers + 32;        // plus the producer warp
constexpr int kCeVecs = 8;  // 16-byte vectors per consumer: V <= 32768 (bf16), 16384 (fp32)
constexpr int kCeMaxStages = 16;
constexpr int kCeRingBytes = 196608;  // shared memory for the row ring
constexpr int kCeBar = 1;             // named barrier of the consumer warps
constexpr unsigned kCeFull = 0xffffffffu;

struct ChunkSummary {
  int32_t first_id, last_id;
  int32_t cnt_first, cnt_last;  // loss tokens of the first / last run inside the chunk
  int32_t single;               // the chunk is one run
  int32_t tot_first, tot_last;  // totals of those runs over the whole row
};

__global__ void __launch_bounds__(kRunThreads)
run_count_kernel(const int32_t* __restrict__ seg, const int32_t* __restrict__ targets,
                 int64_t S, int64_t V, int32_t* __restrict__ run_n, int32_t* __restrict__ n_samples) {
  __shared__ ChunkSummary cs[kRunThreads];
  __shared__ int32_t block_samples;
  const int64_t b = blockIdx.x;
  const int tid = threadIdx.x;
  const int64_t chunk = (S + kRunThreads - 1) / kRunThreads;
  const int64_t t0 = (int64_t)tid * chunk, t1 = t0 + chunk < S ? t0 + chunk : S;
  const int32_t* sg = seg ? seg + b * S : nullptr;
  const int32_t* tg = targets + b * S;
  auto id_of = [&](int64_t t) { return sg ? sg[t] : 0; };
  // the predicate of ce_weight: a target outside [0, V) carries no loss
  auto loss_tok = [&](int64_t t) {
    const int32_t y = tg[t];
    return y >= 0 && y < V && id_of(t) >= 0 ? 1 : 0;
  };
  if (tid == 0) block_samples = 0;
  ChunkSummary c{};
  if (t0 < t1) {
    // one forward pass whose loads do not wait on the previous token: the
    // first run's loss tokens, whether the chunk is one run, the last run's
    int32_t cur_id = id_of(t0), cur_cnt = 0;
    bool in_first = true;
#pragma unroll 8
    for (int64_t t = t0; t < t1; ++t) {
      const int32_t id = id_of(t);
      const int32_t lt = loss_tok(t);
      if (id != cur_id) {
        if (in_first) c.cnt_first = cur_cnt;
        in_first = false;
        cur_id = id;
        cur_cnt = 0;
      }
      cur_cnt += lt;
    }
    if (in_first) c.cnt_first = cur_cnt;
    c.first_id = id_of(t0);
    c.last_id = cur_id;
    c.single = in_first;
    c.cnt_last = cur_cnt;
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

// Max / sum of one value per consumer thread over the consumer warps.
__device__ __forceinline__ float consumers_max(float v, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(kCeFull, v, o));
  sm100::named_bar_sync(kCeBar, kCeConsumers);
  if (lane == 0) red[warp] = v;
  sm100::named_bar_sync(kCeBar, kCeConsumers);
  v = red[0];
#pragma unroll
  for (int i = 1; i < kCeConsumerWarps; ++i) v = fmaxf(v, red[i]);
  return v;
}

__device__ __forceinline__ float consumers_sum(float v, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(kCeFull, v, o);
  sm100::named_bar_sync(kCeBar, kCeConsumers);
  if (lane == 0) red[warp] = v;
  sm100::named_bar_sync(kCeBar, kCeConsumers);
  v = 0.f;
#pragma unroll
  for (int i = 0; i < kCeConsumerWarps; ++i) v += red[i];
  return v;
}

// Weight of token t: 1 / (n * samples) for a loss token, else 0.  A target
// outside the vocabulary counts as "no loss" (never read out of range).
__device__ __forceinline__ float ce_weight(int32_t y, const int32_t* run_n, int32_t ns, int64_t V,
                                           int64_t t) {
  const int32_t n = run_n[t];
  return (y >= 0 && y < V && n > 0 && ns > 0) ? 1.f / ((float)n * (float)ns) : 0.f;
}

// A 16-byte vector of logits as floats, and gradients back into one.
constexpr float kCeLog2e = 1.4426950408889634f;
template <typename T> struct CeVec;
template <> struct CeVec<__nv_bfloat16> {
  __device__ static void unpack(const uint4& r, float (&x)[8]) {
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {  // element 2k in the low half of word k
      x[2 * k] = __uint_as_float(w[k] << 16);
      x[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
    }
  }
  __device__ static uint4 pack(const float (&g)[8]) {
    return make_uint4(sm100::pack_bf16(g[0], g[1]), sm100::pack_bf16(g[2], g[3]),
                      sm100::pack_bf16(g[4], g[5]), sm100::pack_bf16(g[6], g[7]));
  }
  // running max over the vector, on the packed pairs (exact for bf16)
  __device__ static void max_into(const uint4& r, __nv_bfloat162& m) {
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) m = __hmax2(m, *reinterpret_cast<const __nv_bfloat162*>(&w[k]));
  }
};
template <> struct CeVec<float> {
  __device__ static void unpack(const uint4& r, float (&x)[4]) {
    x[0] = __uint_as_float(r.x);
    x[1] = __uint_as_float(r.y);
    x[2] = __uint_as_float(r.z);
    x[3] = __uint_as_float(r.w);
  }
  __device__ static uint4 pack(const float (&g)[4]) {
    return make_uint4(__float_as_uint(g[0]), __float_as_uint(g[1]), __float_as_uint(g[2]),
                      __float_as_uint(g[3]));
  }
  __device__ static void max_into(const uint4& r, float& m) {
    m = fmaxf(fmaxf(m, __uint_as_float(r.x)), __uint_as_float(r.y));
    m = fmaxf(fmaxf(m, __uint_as_float(r.z)), __uint_as_float(r.w));
  }
};
__device__ __forceinline__ float max_value(const __nv_bfloat162& m) {
  return fmaxf(__low2float(m), __high2float(m));
}
__device__ __forceinline__ float max_value(float m) { return m; }
__device__ __forceinline__ void max_init(__nv_bfloat162& m) {
  m = __floats2bfloat162_rn(-INFINITY, -INFINITY);
}
__device__ __forceinline__ void max_init(float& m) { m = -INFINITY; }

// Rows t = blockIdx.x + k * gridDim.x, k = 0, 1, ...: row k goes through
// stage k % nst of the ring.  Stage s has a FULL barrier (one producer
// arrival, plus the row's bytes when it carries a loss) and an EMPTY barrier
// (one arrival per consumer warp once the row is in registers).  Every wait
// is bounded; a wait that runs out records LWM_ERR_TIMEOUT in *status and all
// roles leave their loops, and the CTA waits (bounded) for copies still in
// flight before it exits.
template <typename T, int NV>
__global__ void __launch_bounds__(kCeThreads, 1)
ce_kernel(const T* __restrict__ logits, const int32_t* __restrict__ targets,
          const int32_t* __restrict__ run_n, const int32_t* __restrict__ n_samples, int64_t n,
          int64_t V, int nst, uint32_t stage_bytes, float* __restrict__ term,
          T* __restrict__ dlogits, DeviceStatus* status) {
  constexpr int E = 16 / sizeof(T);
  extern __shared__ __align__(128) uint8_t ce_ring[];
  __shared__ __align__(8) uint64_t full_bar[kCeMaxStages];
  __shared__ __align__(8) uint64_t empty_bar[kCeMaxStages];
  __shared__ float slot_w[kCeMaxStages];
  __shared__ int32_t slot_y[kCeMaxStages];
  __shared__ float red[kCeConsumerWarps];
  __shared__ int s_ok[2];
  __shared__ int s_abort;
  __shared__ long long s_consumed;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t G = gridDim.x;
  const uint32_t row_bytes = (uint32_t)(V * (int64_t)sizeof(T));
  const int64_t nvec = V / E;  // V is a multiple of E (checked by the caller)
  const uint32_t ring = (uint32_t)__cvta_generic_to_shared(ce_ring);
  auto full = [&](int s) { return (uint32_t)__cvta_generic_to_shared(&full_bar[s]); };
  auto empty = [&](int s) { return (uint32_t)__cvta_generic_to_shared(&empty_bar[s]); };
  if (tid == 0) {
    s_abort = 0;
    s_consumed = 0;
    for (int s = 0; s < nst; ++s) {
      sm100::mbar_init(full(s), 1);
      sm100::mbar_init(empty(s), kCeConsumerWarps);
    }
    sm100::fence_mbar_init();
  }
  __syncthreads();
  const sm100::Abort ab{&s_abort, status};
  long long handed = 0;  // rows the producer put into the ring

  if (warp == kCeConsumerWarps) {
    // producer: weights of 32 upcoming rows at a time, one per lane
    const int32_t ns = *n_samples;
    long long k = 0;
    bool ok = true;
    for (int64_t base = blockIdx.x; ok && base < n; base += 32 * G) {
      const int64_t mine = base + (int64_t)lane * G;
      const int32_t yl = mine < n ? targets[mine] : -1;
      const float wl = mine < n ? ce_weight(yl, run_n, ns, V, mine) : 0.f;
      for (int l = 0; l < 32; ++l) {
        const int64_t t = base + (int64_t)l * G;
        if (t >= n) break;
        const float w = __shfl_sync(kCeFull, wl, l);
        const int32_t y = __shfl_sync(kCeFull, yl, l);
        const int s = (int)(k % nst);
        const uint32_t par = (uint32_t)((k / nst) & 1) ^ 1u;
        int good = 1;
        if (lane == 0) {
          good = sm100::mbar_wait(empty(s), par, ab, 1);
          if (good) {
            slot_w[s] = w;
            slot_y[s] = y;
            if (w != 0.f) {
              sm100::mbar_expect_tx(full(s), row_bytes);
              sm100::bulk_load(ring + (uint32_t)s * stage_bytes, logits + t * V, row_bytes,
                               full(s));
            } else {
              sm100::mbar_arrive(full(s));
            }
          }
        }
        good = __shfl_sync(kCeFull, good, 0);
        if (!good) {
          ok = false;
          break;
        }
        ++k;
      }
    }
    handed = k;
  } else {
    // consumers
    long long k = 0;
    for (int64_t t = blockIdx.x; t < n; t += G, ++k) {
      const int s = (int)(k % nst);
      const uint32_t par = (uint32_t)((k / nst) & 1);
      if (tid == 0) s_ok[k & 1] = sm100::mbar_wait(full(s), par, ab, 2);
      sm100::named_bar_sync(kCeBar, kCeConsumers);
      if (!s_ok[k & 1]) break;
      // the phase is complete (thread 0 saw it) and cannot move on before this
      // warp frees the stage: each thread observes it for the copy's bytes
      for (int it = 0; it < (1 << 20) && !sm100::mbar_try(full(s), par); ++it) {
      }
      const float w = slot_w[s];
      const uint4* buf = reinterpret_cast<const uint4*>(ce_ring + (size_t)s * stage_bytes);
      if (w == 0.f) {  // no loss here: zero gradient row
        __syncwarp();
        if (lane == 0) sm100::mbar_arrive(empty(s));
        if (dlogits) {
          uint4* out = reinterpret_cast<uint4*>(dlogits + t * V);
          for (int64_t i = tid; i < nvec; i += kCeConsumers) out[i] = make_uint4(0, 0, 0, 0);
        }
        if (tid == 0) term[t] = 0.f;
        continue;
      }
      const int32_t y = slot_y[s];
      // the target logit, read by the thread that writes the loss term before
      // its warp frees the stage
      const float zy = tid == 0 ? to_f32(reinterpret_cast<const T*>(buf)[y]) : 0.f;
      uint4 raw[NV];
#pragma unroll
      for (int j = 0; j < NV; ++j) {
        const int i = tid + j * kCeConsumers;
        raw[j] = i < nvec ? buf[i] : make_uint4(0, 0, 0, 0);
      }
      __syncwarp();
      if (lane == 0) sm100::mbar_arrive(empty(s));  // the row is in registers
      using V16 = CeVec<T>;
      using MaxT = typename std::conditional<sizeof(T) == 2, __nv_bfloat162, float>::type;
      MaxT mv;
      max_init(mv);
#pragma unroll
      for (int j = 0; j < NV; ++j)
        if (tid + j * kCeConsumers < nvec) V16::max_into(raw[j], mv);
      const float mx = consumers_max(max_value(mv), red);
      const float m2 = mx * kCeLog2e;
      float s0 = 0.f, s1 = 0.f;
#pragma unroll
      for (int j = 0; j < NV; ++j) {
        if (tid + j * kCeConsumers < nvec) {
          float x[E];
          V16::unpack(raw[j], x);
#pragma unroll
          for (int u = 0; u < E; u += 2) {
            s0 += sm100::fast_exp2(fmaf(x[u], kCeLog2e, -m2));
            s1 += sm100::fast_exp2(fmaf(x[u + 1], kCeLog2e, -m2));
          }
        }
      }
      const float sum = consumers_sum(s0 + s1, red);
      const float lse = mx + __logf(sum);
      if (tid == 0) term[t] = w * (lse - zy);
      if (dlogits) {
        const float l2 = lse * kCeLog2e;
        const int yv = y / E, yu = y % E;
        uint4* out = reinterpret_cast<uint4*>(dlogits + t * V);
#pragma unroll
        for (int j = 0; j < NV; ++j) {
          const int i = tid + j * kCeConsumers;
          if (i < nvec) {
            float x[E];
            V16::unpack(raw[j], x);
#pragma unroll
            for (int u = 0; u < E; ++u) x[u] = w * sm100::fast_exp2(fmaf(x[u], kCeLog2e, -l2));
            if (i == yv) {
#pragma unroll
              for (int u = 0; u < E; ++u) x[u] -= u == yu ? w : 0.f;
            }
            out[i] = V16::pack(x);
          }
        }
      }
    }
    if (tid == 0) s_consumed = k;
  }
  __syncthreads();
  // rows handed out but never taken (a wait gave up): their copies may still
  // be in flight into this CTA's shared memory, so wait for them (bounded)
  if (warp == kCeConsumerWarps && lane == 0) {
    for (long long j = s_consumed; j < handed; ++j) {
      const int s = (int)(j % nst);
      const uint32_t par = (uint32_t)((j / nst) & 1);
      const long long t0 = clock64();
      while (!sm100::mbar_try(full(s), par) && clock64() - t0 < sm100::kWaitCycles) {
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

// Workspace: status word (256 bytes), sample counter (256), run_n, terms.
size_t packed_ce_workspace_bytes(int64_t B, int64_t S) {
  const size_t n = (size_t)B * S;
  return 512 + ((n * 4 + 255) / 256) * 256 * 2;
}

int64_t packed_ce_max_vocab(int dtype) {
  return (int64_t)kCeConsumers * kCeVecs * (dtype == LWM_DTYPE_BF16 ? 8 : 4);
}

cudaError_t launch_packed_ce(int64_t B, int64_t S, int64_t V, int dtype, const void* logits,
                             const int32_t* targets, const int32_t* seg, float* loss,
                             void* dlogits, void* ws, cudaStream_t st) {
  const size_t n = (size_t)B * S;
  char* base = static_cast<char*>(ws);
  DeviceStatus* status = reinterpret_cast<DeviceStatus*>(base);
  int32_t* n_samples = reinterpret_cast<int32_t*>(base + 256);
  int32_t* run_n = reinterpret_cast<int32_t*>(base + 512);
  float* term = reinterpret_cast<float*>(base + 512 + ((n * 4 + 255) / 256) * 256);
  cudaError_t e = cudaMemsetAsync(base, 0, 512, st);  // status and sample counter
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return e;
  const size_t elt = dtype == LWM_DTYPE_BF16 ? 2 : 4;
  const uint32_t stage_bytes = (uint32_t)(((size_t)V * elt + 127) / 128 * 128);
  const int nst = (int)std::min<size_t>(kCeMaxStages, kCeRingBytes / stage_bytes);
  const size_t smem = (size_t)nst * stage_bytes;
  const unsigned grid = (unsigned)std::min<size_t>(n, (size_t)sms);
  run_count_kernel<<<(unsigned)B, kRunThreads, 0, st>>>(seg, targets, S, V, run_n, n_samples);
  if (dtype == LWM_DTYPE_BF16) {
    auto kern = ce_kernel<__nv_bfloat16, kCeVecs>;
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) !=
        cudaSuccess)
      return e;
    kern<<<grid, kCeThreads, smem, st>>>(static_cast<const __nv_bfloat16*>(logits), targets,
                                         run_n, n_samples, (int64_t)n, V, nst, stage_bytes, term,
                                         static_cast<__nv_bfloat16*>(dlogits), status);
  } else {
    auto kern = ce_kernel<float, kCeVecs>;
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) !=
        cudaSuccess)
      return e;
    kern<<<grid, kCeThreads, smem, st>>>(static_cast<const float*>(logits), targets, run_n,
                                         n_samples, (int64_t)n, V, nst, stage_bytes, term,
                                         static_cast<float*>(dlogits), status);
  }
  loss_sum_kernel<<<1, 1024, 0, st>>>(term, (int64_t)n, loss);
  note_launches(3);
  return cudaGetLastError();
}

}  // namespace lwm
