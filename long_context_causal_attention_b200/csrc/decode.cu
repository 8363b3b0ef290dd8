// Decode attention: T new query tokens against a key/value cache of S tokens
// (bf16, head_dim 128), with the packing mask and RoPE of the training path.
//
// Generation over a million-token context (LWM research note, sections
// "模型架构" and "Infra"): the new tokens are the last T positions of each
// row, their own keys and values already appended to the cache, and query t
// at position p_t = S - T + t attends exactly as row p_t of the forward pass.
// The cache holds rotated keys (R(j) k_j, as lwm_rope_apply writes them); the
// queries arrive un-rotated and are turned here, in fp32, at their positions.
//
// Work per (b, h) is one pass over the cache rows the new tokens may see, so
// the path is bound by HBM bandwidth, not arithmetic (about one multiply-add
// per byte): CUDA cores, no tensor-core reshaping.  Split-KV in two kernels:
//   decode_partial_kernel  one CTA per (512-key chunk, head, row): scores,
//                          a chunk-local softmax (max m, sum l in the log2
//                          domain) and the unnormalised sum of p * v, merged
//                          over the CTA's eight warps, written to workspace;
//                          chunks whose 128-token tiles hold none of the
//                          queries' segment ids are never read.
//   decode_merge_kernel    one CTA per (new token, head, row): the exact
//                          log-sum-exp merge of all chunk partials, O / L in
//                          bf16 and LSE = (M + log2 L) ln 2.
// Lane mapping inside a warp: lane l owns head dimensions 4l .. 4l+3, so a
// cache row of one head (256 bytes) is one coalesced 8-byte load per lane.
// A batch of NP / TG keys x TG queries gives NP (16 or 32) partial dot
// products per lane; a butterfly folds them so that lane l ends with the
// full product of pair l / R, R = 32 / NP (key (l / R) / TG, query
// (l / R) % TG).
#include <cuda_bf16.h>

#include "common.cuh"
#include "internal.h"

namespace lwm {

namespace {

constexpr int kD = 128;
constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kKeysPerWarp = kDecodeChunk / kWarps;  // 64
constexpr float kLn2 = 0.6931471805599453f;

struct DecParams {
  const __nv_bfloat16* q;  // [B, T, H, D] un-rotated
  const __nv_bfloat16* k;  // [B, S, H, D] rotated cache
  const __nv_bfloat16* v;  // [B, S, H, D]
  const int32_t* seg;      // [B, S] or null
  const int32_t* tmin;     // [B, n_tiles]
  const int32_t* tmax;
  float* part_ml;          // [B, H, T, n_chunks, 2]: chunk max and sum, log2 domain
  float* part_o;           // [B, H, T, n_chunks, D]: unnormalised sum of p * v
  __nv_bfloat16* o;        // [B, T, H, D]
  float* lse;              // [B, H, T]
  int64_t S;
  int T, H, n_chunks, n_tiles;
  float scale_log2;
  int causal, rotate;
  double log2_theta;
};

__device__ __forceinline__ float4 bf16x4(uint2 u) {
  const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&u.x);
  const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&u.y);
  const float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
  return make_float4(fa.x, fa.y, fb.x, fb.y);
}

__device__ __forceinline__ uint2 ldg8(const __nv_bfloat16* p) {
  return __ldg(reinterpret_cast<const uint2*>(p));
}

// Element `i` (runtime, < TG) of a TG-element register array without local
// memory: a chain of selects the compiler unrolls.
template <int TG, typename X>
__device__ __forceinline__ X pick(const X (&a)[TG], int i) {
  X r = a[0];
#pragma unroll
  for (int t = 1; t < TG; ++t) r = i == t ? a[t] : r;
  return r;
}

template <int TG, int NP>
__global__ void __launch_bounds__(kThreads, 2)
decode_partial_kernel(const DecParams p) {
  constexpr int KB = NP / TG;  // keys per batch
  constexpr int R = 32 / NP;   // lanes that end with the same pair
  __shared__ float sm_m[kWarps][TG], sm_l[kWarps][TG];
  __shared__ float sm_o[kWarps][TG][kD];
  const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t k0 = (int64_t)c * kDecodeChunk;
  const size_t rowS = (size_t)b * p.S;
  const int32_t* segrow = p.seg ? p.seg + rowS : nullptr;

  for (int t0 = 0; t0 < p.T; t0 += TG) {
    // ---- this lane's four dimensions of each rotated query of the group ----
    float qv[TG][4];
    int32_t segq[TG];
    int64_t posq[TG];
#pragma unroll
    for (int tt = 0; tt < TG; ++tt) {
      const int t = t0 + tt;
      const bool valid = t < p.T;
      posq[tt] = p.S - p.T + (valid ? t : 0);
      segq[tt] = valid ? (segrow ? segrow[posq[tt]] : 0) : -1;
      float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
      if (valid) x = bf16x4(ldg8(p.q + (((size_t)b * p.T + t) * p.H + h) * kD + 4 * lane));
      if (p.rotate) {
        float c0, s0, c1, s1;
        rope_cos_sin_w(posq[tt], rope_freq(2 * lane, kD, p.log2_theta), &c0, &s0);
        rope_cos_sin_w(posq[tt], rope_freq(2 * lane + 1, kD, p.log2_theta), &c1, &s1);
        const float4 y = make_float4(x.x * c0 - x.y * s0, x.x * s0 + x.y * c0,
                                     x.z * c1 - x.w * s1, x.z * s1 + x.w * c1);
        x = y;
      }
      qv[tt][0] = x.x;
      qv[tt][1] = x.y;
      qv[tt][2] = x.z;
      qv[tt][3] = x.w;
    }
    // ---- skip the chunk when none of its tiles holds a query's segment ----
    bool any = true;
    if (p.seg) {
      any = false;
      for (int tile = (int)(k0 / kTile); tile < p.n_tiles && (int64_t)tile * kTile < k0 + kDecodeChunk;
           ++tile) {
        const int32_t mn = p.tmin[(size_t)b * p.n_tiles + tile];
        const int32_t mx = p.tmax[(size_t)b * p.n_tiles + tile];
#pragma unroll
        for (int tt = 0; tt < TG; ++tt)
          any |= segq[tt] >= 0 && mx >= 0 && mn <= segq[tt] && segq[tt] <= mx;
      }
    }
    float m[TG], l[TG], acc[TG][4];
#pragma unroll
    for (int tt = 0; tt < TG; ++tt) {
      m[tt] = -INFINITY;
      l[tt] = 0.f;
      acc[tt][0] = acc[tt][1] = acc[tt][2] = acc[tt][3] = 0.f;
    }
    if (any) {
      const int my_t = (lane / R) % TG;  // query of the pair this lane ends with
      const int my_j = (lane / R) / TG;  // key of that pair within the batch
      const int32_t my_seg = pick<TG>(segq, my_t);
      const int64_t my_pos = pick<TG>(posq, my_t);
      for (int kb = 0; kb < kKeysPerWarp; kb += KB) {
        const int64_t kbase = k0 + warp * kKeysPerWarp + kb;
        if (kbase >= p.S) break;
        // the batch's key and value rows in one burst of loads (more bytes
        // in flight per warp), then NP partial products per lane, folded
        float d[NP];
        uint2 vr[KB];
        {
          uint2 kr[KB];
#pragma unroll
          for (int j = 0; j < KB; ++j) {
            const int64_t key = kbase + j;
            const size_t off = ((rowS + key) * p.H + h) * kD + 4 * lane;
            kr[j] = key < p.S ? ldg8(p.k + off) : make_uint2(0u, 0u);
            vr[j] = key < p.S ? ldg8(p.v + off) : make_uint2(0u, 0u);
          }
#pragma unroll
          for (int j = 0; j < KB; ++j) {
            const float4 kf = bf16x4(kr[j]);
#pragma unroll
            for (int tt = 0; tt < TG; ++tt)
              d[j * TG + tt] = qv[tt][0] * kf.x + qv[tt][1] * kf.y + qv[tt][2] * kf.z +
                               qv[tt][3] * kf.w;
          }
        }
#pragma unroll
        for (int off = 16, n = NP; off >= R; off >>= 1, n >>= 1) {
          const bool upper = (lane & off) != 0;
#pragma unroll
          for (int i = 0; i < n / 2; ++i) {
            const float send = upper ? d[i] : d[i + n / 2];
            const float keep = upper ? d[i + n / 2] : d[i];
            d[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
          }
        }
#pragma unroll
        for (int off = R / 2; off >= 1; off >>= 1) d[0] += __shfl_xor_sync(0xffffffffu, d[0], off);
        const int64_t key = kbase + my_j;
        bool ok = key < p.S && my_seg >= 0 && (!p.causal || key <= my_pos);
        if (ok && segrow) ok = __ldg(segrow + key) == my_seg;
        const float sv = ok ? d[0] * p.scale_log2 : -INFINITY;
        // online softmax per query (the lanes of one query differ in bits >= log2 TG)
        float bm = sv;
#pragma unroll
        for (int off = R * TG; off < 32; off <<= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, off));
        const float mo = pick<TG>(m, my_t);
        const float mn = fmaxf(mo, bm);
        const float corr = mn == -INFINITY ? 1.f : exp2f(mo - mn);
        const float pv = ok ? exp2f(sv - mn) : 0.f;
        float ps = pv;
#pragma unroll
        for (int off = R * TG; off < 32; off <<= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
#pragma unroll
        for (int tt = 0; tt < TG; ++tt) {
          const float ct = __shfl_sync(0xffffffffu, corr, tt * R);
          m[tt] = __shfl_sync(0xffffffffu, mn, tt * R);
          l[tt] = l[tt] * ct + __shfl_sync(0xffffffffu, ps, tt * R);
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[tt][e] *= ct;
        }
        // p * v
#pragma unroll
        for (int j = 0; j < KB; ++j) {
          const float4 vf = bf16x4(vr[j]);
#pragma unroll
          for (int tt = 0; tt < TG; ++tt) {
            const float pj = __shfl_sync(0xffffffffu, pv, (j * TG + tt) * R);
            acc[tt][0] = fmaf(pj, vf.x, acc[tt][0]);
            acc[tt][1] = fmaf(pj, vf.y, acc[tt][1]);
            acc[tt][2] = fmaf(pj, vf.z, acc[tt][2]);
            acc[tt][3] = fmaf(pj, vf.w, acc[tt][3]);
          }
        }
      }
    }
    // ---- merge the eight warps of the CTA, write the chunk partial ----
    if (lane < TG) {
      sm_m[warp][lane] = pick<TG>(m, lane);
      sm_l[warp][lane] = pick<TG>(l, lane);
    }
#pragma unroll
    for (int tt = 0; tt < TG; ++tt)
      *reinterpret_cast<float4*>(&sm_o[warp][tt][4 * lane]) =
          make_float4(acc[tt][0], acc[tt][1], acc[tt][2], acc[tt][3]);
    __syncthreads();
    for (int idx = threadIdx.x; idx < TG * kD; idx += kThreads) {
      const int tt = idx / kD, dd = idx % kD;
      const int t = t0 + tt;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) M = fmaxf(M, sm_m[w][tt]);
      float L = 0.f, O = 0.f;
      if (M != -INFINITY) {
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
          const float f = sm_m[w][tt] == -INFINITY ? 0.f : exp2f(sm_m[w][tt] - M);
          L += sm_l[w][tt] * f;
          O += sm_o[w][tt][dd] * f;
        }
      }
      if (t < p.T) {
        const size_t pi = (((size_t)b * p.H + h) * p.T + t) * p.n_chunks + c;
        p.part_o[pi * kD + dd] = O;
        if (dd == 0) {
          p.part_ml[2 * pi] = M;
          p.part_ml[2 * pi + 1] = L;
        }
      }
    }
    __syncthreads();
  }
}

constexpr int kMergeSlices = 8;  // chunk slices per merge CTA (one warp group of 128 each)

__global__ void __launch_bounds__(kD * kMergeSlices) decode_merge_kernel(const DecParams p) {
  __shared__ float red[kD * kMergeSlices / 32];
  __shared__ float part[kMergeSlices][kD + 1];
  const int t = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, dd = tid % kD, slice = tid / kD;
  const int warp = tid >> 5, lane = tid & 31;
  constexpr int kWarpsM = kD * kMergeSlices / 32;
  const size_t base = (((size_t)b * p.H + h) * p.T + t) * p.n_chunks;
  const float* ml = p.part_ml + 2 * base;
  // M = max over chunks
  float M = -INFINITY;
  for (int c = tid; c < p.n_chunks; c += kD * kMergeSlices) M = fmaxf(M, ml[2 * c]);
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  if (lane == 0) red[warp] = M;
  __syncthreads();
  M = red[0];
#pragma unroll
  for (int w = 1; w < kWarpsM; ++w) M = fmaxf(M, red[w]);
  // this slice's share of L and of O[dd]
  float L = 0.f, O = 0.f;
  if (M != -INFINITY) {
#pragma unroll 4
    for (int c = slice; c < p.n_chunks; c += kMergeSlices) {
      const float mc = ml[2 * c];
      const float f = mc == -INFINITY ? 0.f : exp2f(mc - M);
      L += ml[2 * c + 1] * f;
      O += p.part_o[(base + c) * kD + dd] * f;
    }
  }
  part[slice][dd] = O;
  if (dd == 0) part[slice][kD] = L;
  __syncthreads();
  if (slice != 0) return;
  O = 0.f;
  L = 0.f;
#pragma unroll
  for (int sl = 0; sl < kMergeSlices; ++sl) {
    O += part[sl][dd];
    L += part[sl][kD];
  }
  const size_t orow = (((size_t)b * p.T + t) * p.H + h) * kD;
  if (L > 0.f) {
    p.o[orow + dd] = __float2bfloat16_rn(O / L);
    if (dd == 0) p.lse[((size_t)b * p.H + h) * p.T + t] = (M + log2f(L)) * kLn2;
  } else {
    p.o[orow + dd] = __float2bfloat16_rn(0.f);
    if (dd == 0) p.lse[((size_t)b * p.H + h) * p.T + t] = -INFINITY;
  }
}

}  // namespace

cudaError_t launch_decode(const Problem& pb, const Workspace& ws, int64_t n_new, const void* q,
                          const void* k_cache, const void* v_cache, void* o, float* lse,
                          cudaStream_t st) {
  DecParams p{};
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k = static_cast<const __nv_bfloat16*>(k_cache);
  p.v = static_cast<const __nv_bfloat16*>(v_cache);
  p.seg = pb.seg;
  p.tmin = ws.tile_min;
  p.tmax = ws.tile_max;
  p.part_ml = ws.dec_ml;
  p.part_o = ws.dec_o;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.S = pb.S;
  p.T = (int)n_new;
  p.H = (int)pb.H;
  p.n_chunks = (int)((pb.S + kDecodeChunk - 1) / kDecodeChunk);
  p.n_tiles = (int)pb.n_tiles;
  p.scale_log2 = pb.scale * 1.4426950408889634f;
  p.causal = pb.causal;
  p.rotate = pb.theta > 0.0;
  p.log2_theta = p.rotate ? log2(pb.theta) : 0.0;
  const dim3 g1((unsigned)p.n_chunks, (unsigned)pb.H, (unsigned)pb.B);
  if (n_new == 1)
    decode_partial_kernel<1, 16><<<g1, kThreads, 0, st>>>(p);
  else if (n_new == 2)
    decode_partial_kernel<2, 32><<<g1, kThreads, 0, st>>>(p);
  else
    decode_partial_kernel<4, 32><<<g1, kThreads, 0, st>>>(p);
  const dim3 g2((unsigned)n_new, (unsigned)pb.H, (unsigned)pb.B);
  decode_merge_kernel<<<g2, kD * kMergeSlices, 0, st>>>(p);
  note_launches(2);
  return cudaGetLastError();
}

}  // namespace lwm
