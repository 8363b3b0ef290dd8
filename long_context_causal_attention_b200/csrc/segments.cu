// Segment-id prepass for masked sequence packing.
//
// LWM research note, section "训练方法", Masked Sequence Packing: samples
// packed into one row attend only to themselves.  Per 128-token tile this
// records the smallest and largest non-negative segment id (tile_min is set
// to -1 instead when the tile holds any padding token, id < 0; tile_max is
// -1 when the tile holds no valid token).  Two tiles can only share an
// allowed pair when their id ranges intersect, so every other tile pair is
// skipped without being loaded, and a tile pair is free of masking inside
// when all four bounds are the same non-negative id.  From the bounds it also derives,
// per query tile, the first key tile it may need (q_lo) and, per key tile, the
// last query tile it may feed (k_hi).  Both are sound for any ids; for ids in
// contiguous runs (what packing produces) they are tight.
#include <climits>

#include "common.cuh"
#include "internal.h"

namespace lwm {
namespace {

__global__ void tile_bounds_kernel(const int32_t* __restrict__ seg, int64_t B, int64_t S,
                                   int64_t n_tiles, int32_t* __restrict__ tmin,
                                   int32_t* __restrict__ tmax) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= B * n_tiles) return;
  const int64_t b = idx / n_tiles, t = idx % n_tiles;
  const int64_t i0 = t * kTile, i1 = min(S, i0 + kTile);
  int32_t lo = INT_MAX, hi = -1;
  bool pad = false;
  const int32_t* row = seg + b * S;
  for (int64_t i = i0; i < i1; ++i) {
    const int32_t s = row[i];
    if (s >= 0) {
      lo = min(lo, s);
      hi = max(hi, s);
    } else {
      pad = true;
    }
  }
  tmin[idx] = (pad || hi < 0) ? -1 : lo;
  tmax[idx] = hi;
}

__device__ __forceinline__ bool meet(int32_t a0, int32_t a1, int32_t b0, int32_t b1) {
  return a1 >= 0 && b1 >= 0 && a0 <= b1 && b0 <= a1;
}

// q bounds (tmin, tmax) describe the query tiles, k bounds the key tiles
// (the same arrays unless the keys carry their own segment ids).
__global__ void tile_ranges_kernel(const int32_t* __restrict__ tmin, const int32_t* __restrict__ tmax,
                                   const int32_t* __restrict__ ktmin,
                                   const int32_t* __restrict__ ktmax, int64_t B, int64_t n_tiles,
                                   int causal, int32_t* __restrict__ q_lo,
                                   int32_t* __restrict__ k_hi) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= B * n_tiles) return;
  const int64_t b = idx / n_tiles, t = idx % n_tiles;
  const int32_t* mn = tmin + b * n_tiles;
  const int32_t* mx = tmax + b * n_tiles;
  const int32_t* kmn = ktmin + b * n_tiles;
  const int32_t* kmx = ktmax + b * n_tiles;
  // first key tile for query tile t
  const int64_t jmax = causal ? t : n_tiles - 1;
  int64_t lo = jmax + 1;
  for (int64_t j = 0; j <= jmax; ++j) {
    if (meet(mn[t], mx[t], kmn[j], kmx[j])) { lo = j; break; }
  }
  q_lo[idx] = (int32_t)lo;
  // last query tile for key tile t
  const int64_t imin = causal ? t : 0;
  int64_t hi = imin - 1;
  for (int64_t i = n_tiles - 1; i >= imin; --i) {
    if (meet(kmn[t], kmx[t], mn[i], mx[i])) { hi = i; break; }
  }
  k_hi[idx] = (int32_t)hi;
}

}  // namespace

cudaError_t launch_segment_bounds(const Problem& p, const Workspace& ws, cudaStream_t st,
                                  bool ranges) {
  if (!p.seg) return cudaSuccess;
  const int64_t n = p.B * p.n_tiles;
  if (n == 0) return cudaSuccess;
  const int threads = 128;
  const unsigned grid = (unsigned)((n + threads - 1) / threads);
  tile_bounds_kernel<<<grid, threads, 0, st>>>(p.seg, p.B, p.S, p.n_tiles, ws.tile_min, ws.tile_max);
  int launched = 1;
  if (p.kseg != p.seg) {
    tile_bounds_kernel<<<grid, threads, 0, st>>>(p.kseg, p.B, p.S, p.n_tiles, ws.ktile_min,
                                                 ws.ktile_max);
    ++launched;
  }
  if (ranges) {
    tile_ranges_kernel<<<grid, threads, 0, st>>>(ws.tile_min, ws.tile_max, ws.ktile_min,
                                                 ws.ktile_max, p.B, p.n_tiles, p.causal, ws.q_lo,
                                                 ws.k_hi);
    ++launched;
  }
  note_launches(launched);
  return cudaGetLastError();
}

}  // namespace lwm
