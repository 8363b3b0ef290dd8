// Forward attention on the 5th-generation tensor cores (sm_100a), bf16, D=128.
//
// What it computes: exact causal softmax attention with a packing mask
// (LWM research note, "模型架构": exact blockwise attention; "训练方法":
// Masked Sequence Packing), over q and k that the RoPE pre-pass has already
// rotated.  Output O (bf16) and LSE = ln sum exp(s) per row (fp32).
//
// Design (one persistent CTA per SM, 384 threads):
//   warp 0      TMA producer: Q tile pair once per work item, then K_j and V_j
//               for every key tile j the pair needs, through 2-stage rings
//               (K runs one tile ahead of V).
//   warp 1      MMA issuer (one thread): S_t = Q_t K_j^T and O_t += P_t V_j
//               with tcgen05.mma, fp32 accumulators in tensor memory.
//   warp 2      allocates / frees the 512 tensor-memory columns.
//   warps 4-7   softmax for query tile t=0 (one row per thread),
//   warps 8-11  softmax for query tile t=1: read S from TMEM, mask partial
//               tiles, online max/sum in log2 units, write P (bf16) back
//               into the S columns for the PV MMA, rescale O when the
//               running max grows by more than 2^8, then normalise and
//               store O (bf16 through 2 KB of shared memory per warp, so
//               that each store instruction writes whole 64-byte row
//               pieces) and LSE.
// TMEM columns: S_0 [0,128), S_1 [128,256), O_0 [256,384), O_1 [384,512);
// P_t is packed bf16 in the first 64 columns of S_t.
// The MMA issue order ping-pongs the two tiles so one softmax warpgroup
// works while the tensor core runs the other tile's MMAs:
//   S_0(j) S_1(j) | PV_0(j) S_0(j+1) | PV_1(j) S_1(j+1) | ...
// Work items (b, h, pair of 128-row query tiles), in head-major order with
// the costliest pair of each head first, come from a global counter: the
// TMA thread takes the next one when it is ready for it and publishes it to
// the CTA through a 4-slot ring, so the CTAs stay on consecutive items of one
// head and share its K/V through L2.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace lwm {
namespace {

using namespace sm100;

constexpr int kD = 128;
constexpr int kThreads = 384;
constexpr uint32_t kTileBytes = 128 * kD * 2;  // one 128 x 128 bf16 tile = two 16 KB boxes
constexpr uint32_t kBoxBytes = kTileBytes / 2;
constexpr float kRescaleLog2 = 8.0f;  // keep a stale max until the true one is 2^8 larger

// shared memory map (offsets from a 1024-byte aligned base)
constexpr uint32_t OFF_Q = 0;                          // Q_0, Q_1
constexpr uint32_t OFF_K = OFF_Q + 2 * kTileBytes;     // K ring, 2 stages
constexpr uint32_t OFF_V = OFF_K + 2 * kTileBytes;     // V ring, 2 stages
constexpr uint32_t OFF_BAR = OFF_V + 2 * kTileBytes;   // mbarriers
constexpr uint32_t OFF_MISC = OFF_BAR + 256;           // TMEM base, abort flag
constexpr uint32_t OFF_FREQ = OFF_MISC + 64;          // 64 RoPE frequencies, fp64
constexpr uint32_t OFF_STG = OFF_FREQ + 512;          // O epilogue staging, 2 KB per softmax warp
constexpr uint32_t kStgWarpBytes = 32 * 64;           // 32 rows x 32 bf16 columns
constexpr uint32_t kSmemBytes = OFF_STG + 8 * kStgWarpBytes + 1024;  // + alignment slack

// barrier slots (8 bytes each)
enum : uint32_t {
  B_Q_FULL = 0, B_Q_EMPTY = 1,
  B_K_FULL = 2,   // 2 stages
  B_K_EMPTY = 4,  // 2
  B_V_FULL = 6,   // 2
  B_V_EMPTY = 8,  // 2
  B_S_FULL = 10,  // per tile
  B_P_FULL = 12,  // per tile
  B_O_FULL = 14,  // per tile
  B_O_EMPTY = 16, // per tile
  B_FIN = 18,
  B_ITEM_FULL = 19,   // 4 slots
  B_ITEM_EMPTY = 23,  // 4 slots
  B_Q_ROT = 27,       // per tile: the softmax warps rotated Q_t in place
  B_COUNT = 29
};
static_assert(B_COUNT * 8 <= 256, "barrier slots");
constexpr uint32_t kItemSlots = 4;
constexpr uint32_t kSoftmaxWarps = 8;

struct FwdParams {
  const int32_t* seg;    // [B, S] query segment ids, or null
  const int32_t* kseg;   // [B, S] key segment ids (seg unless a block pair)
  const int32_t* tmin;   // [B, nT] query tile bounds (valid when seg != null)
  const int32_t* tmax;
  const int32_t* ktmin;  // [B, nT] key tile bounds
  const int32_t* ktmax;
  const int32_t* q_lo;
  __nv_bfloat16* o;
  float* o32;          // non-null: O is written in fp32 here instead (block partials of a ring)
  float* lse;
  DeviceStatus* status;
  int64_t S;
  int H, B, n_tiles, n_pairs;
  float scale_log2;
  int causal;
  int rotate;          // Q tiles arrive un-rotated: RoPE them in shared memory
  double log2_theta;
};

struct Item {
  int b, h;
  int qt[2];       // query tile index, -1 when past the end
  int lo[2], hi[2];
  int32_t qmin[2], qmax[2];
};

__device__ __forceinline__ bool meet(int32_t a0, int32_t a1, int32_t b0, int32_t b1) {
  return a1 >= 0 && b1 >= 0 && a0 <= b1 && b0 <= a1;
}

__device__ __forceinline__ Item decode(const FwdParams& p, int idx) {
  Item it;
  const int bh = idx / p.n_pairs;
  const int pr = p.n_pairs - 1 - (idx % p.n_pairs);
  it.b = bh / p.H;
  it.h = bh % p.H;
  for (int t = 0; t < 2; ++t) {
    const int qt = 2 * pr + t;
    it.qt[t] = qt < p.n_tiles ? qt : -1;
    it.lo[t] = 0;
    it.hi[t] = -1;
    it.qmin[t] = 0;
    it.qmax[t] = 0;
    if (it.qt[t] < 0) continue;
    const size_t ti = (size_t)it.b * p.n_tiles + qt;
    it.hi[t] = p.causal ? qt : p.n_tiles - 1;
    if (p.seg) {
      it.lo[t] = p.q_lo[ti];
      it.qmin[t] = p.tmin[ti];
      it.qmax[t] = p.tmax[ti];
    }
  }
  return it;
}

__device__ __forceinline__ bool rel(const FwdParams& p, const Item& it, int t, int j) {
  if (it.qt[t] < 0 || j < it.lo[t] || j > it.hi[t]) return false;
  if (!p.seg) return true;
  const size_t kj = (size_t)it.b * p.n_tiles + j;
  return meet(it.qmin[t], it.qmax[t], p.ktmin[kj], p.ktmax[kj]);
}

__device__ __forceinline__ bool rel_any(const FwdParams& p, const Item& it, int j) {
  return rel(p, it, 0, j) || rel(p, it, 1, j);
}

__device__ __forceinline__ int next_any(const FwdParams& p, const Item& it, int j, int jend) {
  for (++j; j <= jend; ++j)
    if (rel_any(p, it, j)) return j;
  return -1;
}

// The next key tile after j that either query tile needs, and which of the
// two need it (rn[t]); the segment bounds of each tile are loaded once.
__device__ __forceinline__ int next_rel2(const FwdParams& p, const Item& it, int j, int jend,
                                         bool (&rn)[2]) {
  for (++j; j <= jend; ++j) {
    bool r0 = it.qt[0] >= 0 && j >= it.lo[0] && j <= it.hi[0];
    bool r1 = it.qt[1] >= 0 && j >= it.lo[1] && j <= it.hi[1];
    if (p.seg && (r0 || r1)) {
      const size_t kj = (size_t)it.b * p.n_tiles + j;
      const int32_t a0 = p.ktmin[kj], a1 = p.ktmax[kj];
      r0 = r0 && meet(it.qmin[0], it.qmax[0], a0, a1);
      r1 = r1 && meet(it.qmin[1], it.qmax[1], a0, a1);
    }
    if (r0 || r1) {
      rn[0] = r0;
      rn[1] = r1;
      return j;
    }
  }
  rn[0] = rn[1] = false;
  return -1;
}

__device__ __forceinline__ void union_range(const Item& it, int* jlo, int* jhi) {
  int lo = 1 << 30, hi = -1;
  for (int t = 0; t < 2; ++t) {
    if (it.qt[t] < 0 || it.lo[t] > it.hi[t]) continue;
    lo = min(lo, it.lo[t]);
    hi = max(hi, it.hi[t]);
  }
  *jlo = lo;
  *jhi = hi;
}

// A wait that ignores the abort flag: used only while draining.
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try(bar, parity)) {
    if (clock64() - t0 > kWaitCycles) return;
  }
}

__global__ void __launch_bounds__(kThreads, 1)
attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  const uint32_t bar0 = base + OFF_BAR;
  auto bar = [&](uint32_t slot) { return bar0 + 8u * slot; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_MISC + 8);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  // work items come from a global counter (greedy, in cost order): the TMA
  // thread takes one and publishes it to the CTA through a 4-slot ring
  volatile int* item_slot = reinterpret_cast<volatile int*>(smem + OFF_MISC + 16);
  int* item_counter = &p.status->item_counter[2];
  const Abort ab{abort_flag, p.status};

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_items = p.B * p.H * p.n_pairs;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(bar(B_Q_FULL), 1);
    mbar_init(bar(B_Q_EMPTY), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(B_K_FULL + s), 1);
      mbar_init(bar(B_K_EMPTY + s), 1);
      mbar_init(bar(B_V_FULL + s), 1);
      mbar_init(bar(B_V_EMPTY + s), 1);
      mbar_init(bar(B_S_FULL + s), 1);
      mbar_init(bar(B_P_FULL + s), 128);
      mbar_init(bar(B_O_FULL + s), 1);
      mbar_init(bar(B_O_EMPTY + s), 128);
    }
    mbar_init(bar(B_FIN), 1);
    for (uint32_t sl = 0; sl < kItemSlots; ++sl) {
      mbar_init(bar(B_ITEM_FULL + sl), 1);
      mbar_init(bar(B_ITEM_EMPTY + sl), 1 + kSoftmaxWarps);
    }
    mbar_init(bar(B_Q_ROT), kSoftmaxWarps / 2);
    mbar_init(bar(B_Q_ROT + 1), kSoftmaxWarps / 2);
    fence_mbar_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  double* freq = reinterpret_cast<double*>(smem + OFF_FREQ);
  if (threadIdx.x >= 128 && threadIdx.x < 128 + kD / 2 && p.rotate)
    freq[threadIdx.x - 128] = rope_freq(threadIdx.x - 128, kD, p.log2_theta);
  if (warp == 2) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // per-stage state the producer keeps for draining after an abort
  uint32_t k_issued = 0, v_issued = 0;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA
    if (lane == 0) {
      uint32_t k_it = 0, v_it = 0;
      int items = 0;
      bool ok = true;
      for (uint32_t pub = 0; ok; ++items) {
        const uint32_t sl = pub % kItemSlots;
        if (pub >= kItemSlots &&
            !mbar_wait(bar(B_ITEM_EMPTY + sl), ((pub / kItemSlots) - 1) & 1, ab, 13)) {
          ok = false;
          break;
        }
        const int idx = atomicAdd(item_counter, 1);
        item_slot[sl] = idx;
        mbar_arrive(bar(B_ITEM_FULL + sl));
        ++pub;
        if (idx >= n_items) break;
        const Item it = decode(p, idx);
        if (items > 0 && !mbar_wait(bar(B_Q_EMPTY), (items - 1) & 1, ab, 1)) { ok = false; break; }
        const int nq = (it.qt[0] >= 0) + (it.qt[1] >= 0);
        mbar_expect_tx(bar(B_Q_FULL), nq * kTileBytes);
        for (int t = 0; t < 2; ++t) {
          if (it.qt[t] < 0) continue;
          const uint32_t dst = base + OFF_Q + t * kTileBytes;
          tma_load_4d(dst, &tm_q, bar(B_Q_FULL), 0, it.h, it.qt[t] * 128, it.b);
          tma_load_4d(dst + kBoxBytes, &tm_q, bar(B_Q_FULL), 64, it.h, it.qt[t] * 128, it.b);
        }
        int jlo, jhi;
        union_range(it, &jlo, &jhi);
        int j = (jlo <= jhi && rel_any(p, it, jlo)) ? jlo : next_any(p, it, jlo, jhi);
        auto load_k = [&](int jj) -> bool {
          const uint32_t s = k_it & 1;
          if (!mbar_wait(bar(B_K_EMPTY + s), ((k_it >> 1) & 1) ^ 1, ab, 2)) return false;
          mbar_expect_tx(bar(B_K_FULL + s), kTileBytes);
          const uint32_t dst = base + OFF_K + s * kTileBytes;
          tma_load_4d(dst, &tm_k, bar(B_K_FULL + s), 0, it.h, jj * 128, it.b);
          tma_load_4d(dst + kBoxBytes, &tm_k, bar(B_K_FULL + s), 64, it.h, jj * 128, it.b);
          ++k_it;
          k_issued = k_it;
          return true;
        };
        auto load_v = [&](int jj) -> bool {
          const uint32_t s = v_it & 1;
          if (!mbar_wait(bar(B_V_EMPTY + s), ((v_it >> 1) & 1) ^ 1, ab, 3)) return false;
          mbar_expect_tx(bar(B_V_FULL + s), kTileBytes);
          const uint32_t dst = base + OFF_V + s * kTileBytes;
          tma_load_4d(dst, &tm_v, bar(B_V_FULL + s), 0, it.h, jj * 128, it.b);
          tma_load_4d(dst + kBoxBytes, &tm_v, bar(B_V_FULL + s), 64, it.h, jj * 128, it.b);
          ++v_it;
          v_issued = v_it;
          return true;
        };
        if (j >= 0 && !load_k(j)) { ok = false; break; }
        while (j >= 0) {
          const int jn = next_any(p, it, j, jhi);
          if (jn >= 0 && !load_k(jn)) { ok = false; break; }
          if (!load_v(j)) { ok = false; break; }
          j = jn;
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA
    if (lane == 0) {
      constexpr uint32_t kIdS = idesc_bf16(128, 128, 0, 0);  // Q (K-major) x K (K-major)
      constexpr uint32_t kIdPV = idesc_bf16(128, 128, 0, 1); // P (TMEM) x V (MN-major)
      uint32_t k_it = 0, v_it = 0, p_cnt[2] = {0, 0}, act[2] = {0, 0}, rot[2] = {0, 0};
      int items = 0;
      bool ok = true;
      const uint32_t sq0 = base + OFF_Q;
      const uint64_t dQ0 = kmajor_desc(sq0), dQ1 = kmajor_desc(sq0 + kTileBytes);
      const uint64_t dK0 = kmajor_desc(base + OFF_K), dK1 = kmajor_desc(base + OFF_K + kTileBytes);
      const uint64_t dV0 = mnmajor_desc(base + OFF_V), dV1 = mnmajor_desc(base + OFF_V + kTileBytes);
      for (uint32_t cons = 0; ok; ++items) {
        const uint32_t sl = cons % kItemSlots;
        if (!mbar_wait(bar(B_ITEM_FULL + sl), (cons / kItemSlots) & 1, ab, 14)) { ok = false; break; }
        const int idx = item_slot[sl];
        mbar_arrive(bar(B_ITEM_EMPTY + sl));
        ++cons;
        if (idx >= n_items) break;
        const Item it = decode(p, idx);
        if (!mbar_wait(bar(B_Q_FULL), items & 1, ab, 4)) { ok = false; break; }
        if (p.rotate) {  // and the softmax warps have rotated the tiles in place
          for (int t = 0; t < 2 && ok; ++t) {
            if (it.qt[t] < 0) continue;
            ok = mbar_wait(bar(B_Q_ROT + t), rot[t] & 1, ab, 24);
            ++rot[t];
          }
          if (!ok) break;
        }
        tc_fence_after();
        int jlo, jhi;
        union_range(it, &jlo, &jhi);
        bool rc[2];  // which query tiles need key tile jc
        const int jc0 = next_rel2(p, it, jlo - 1, jhi, rc);
        int jc = jlo <= jhi ? jc0 : -1;
        bool first_pv[2] = {true, true}, active[2] = {false, false};

        // descriptors precomputed: the issuing thread's work between two
        // products idles the tensor core, so it is kept to a minimum
        auto issue_s = [&](int t) {
          mma_kk128(tmem + (uint32_t)(t * 128), t ? dQ1 : dQ0, (k_it & 1) ? dK1 : dK0, kIdS, 0u);
          mma_commit(bar(B_S_FULL + t));
        };
        auto issue_pv = [&](int t) {
          mma_tm128<false>(tmem + 256u + (uint32_t)(t * 128), tmem + (uint32_t)(t * 128),
                           (v_it & 1) ? dV1 : dV0, kIdPV, first_pv[t] ? 0u : 1u);
          first_pv[t] = false;
        };

        if (jc >= 0) {
          if (!mbar_wait(bar(B_K_FULL + (k_it & 1)), (k_it >> 1) & 1, ab, 5)) { ok = false; break; }
          tc_fence_after();
          for (int t = 0; t < 2; ++t)
            if (rc[t]) issue_s(t);
          mma_commit(bar(B_K_EMPTY + (k_it & 1)));
          ++k_it;
        }
        bool q_released = false;
        while (jc >= 0 && ok) {
          bool rn[2];
          const int jn = next_rel2(p, it, jc, jhi, rn);
          if (jn < 0) {
            // every S of the item is issued: the Q tiles are free once those
            // complete, so the producer loads the next item's Q tiles while
            // this item's last softmax and PV products run
            mma_commit(bar(B_Q_EMPTY));
            q_released = true;
          }
          bool v_ready = false, k_ready = false;
          for (int t = 0; t < 2 && ok; ++t) {
            if (rc[t]) {
              if (!v_ready) {
                if (!mbar_wait(bar(B_V_FULL + (v_it & 1)), (v_it >> 1) & 1, ab, 6)) { ok = false; break; }
                v_ready = true;
              }
              if (first_pv[t] && act[t] > 0) {
                if (!mbar_wait(bar(B_O_EMPTY + t), (act[t] - 1) & 1, ab, 7)) { ok = false; break; }
              }
              if (!mbar_wait(bar(B_P_FULL + t), p_cnt[t] & 1, ab, 8)) { ok = false; break; }
              ++p_cnt[t];
              tc_fence_after();
              issue_pv(t);
              active[t] = true;
            }
            if (jn >= 0 && rn[t]) {
              if (!k_ready) {
                if (!mbar_wait(bar(B_K_FULL + (k_it & 1)), (k_it >> 1) & 1, ab, 9)) { ok = false; break; }
                tc_fence_after();
                k_ready = true;
              }
              issue_s(t);
            }
          }
          if (!ok) break;
          if (k_ready) {
            mma_commit(bar(B_K_EMPTY + (k_it & 1)));
            ++k_it;
          }
          mma_commit(bar(B_V_EMPTY + (v_it & 1)));
          ++v_it;
          jc = jn;
          rc[0] = rn[0];
          rc[1] = rn[1];
        }
        if (!ok) break;
        for (int t = 0; t < 2; ++t) {
          if (active[t]) {
            mma_commit(bar(B_O_FULL + t));
            ++act[t];
          }
        }
        if (!q_released) mma_commit(bar(B_Q_EMPTY));
      }
    }
  } else if (warp >= 4) {
    // -------------------------------------------------------------- softmax
    const int t = (warp - 4) >> 2;          // query tile of this warpgroup
    const int tid = threadIdx.x - 128 - 128 * t;  // 0..127 = TMEM lane = row in tile
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + (uint32_t)(t * 128);
    const uint32_t tO = tmem + lane_base + 256u + (uint32_t)(t * 128);
    uint32_t s_cnt = 0, o_cnt = 0, q_items = 0;
    bool ok = true;
    for (uint32_t cons = 0; ok;) {
      const uint32_t sl = cons % kItemSlots;
      if (!__all_sync(0xffffffffu, mbar_wait(bar(B_ITEM_FULL + sl), (cons / kItemSlots) & 1, ab, 15))) {
        ok = false;
        break;
      }
      const int idx = item_slot[sl];
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_ITEM_EMPTY + sl));
      ++cons;
      if (idx >= n_items) break;
      const Item it = decode(p, idx);
      const uint32_t q_phase = q_items++ & 1;  // Q_FULL completes once per item
      // this warpgroup's query tile: its fields picked once, kept in registers
      const int qt_t = t ? it.qt[1] : it.qt[0];
      const int lo_t = t ? it.lo[1] : it.lo[0], hi_t = t ? it.hi[1] : it.hi[0];
      const int32_t qmin_t = t ? it.qmin[1] : it.qmin[0], qmax_t = t ? it.qmax[1] : it.qmax[0];
      if (qt_t < 0) continue;
      const int64_t row = (int64_t)qt_t * 128 + tid;
      if (p.rotate) {
        // RoPE on this row of the Q tile, in place in shared memory: pair
        // (2i, 2i+1) turns by row * w_i, the angle reduced in fp64 and cos/sin
        // from the fast approximation (absolute error below 1e-6, far under
        // the bf16 rounding of the result)
        if (!__all_sync(0xffffffffu, mbar_wait(bar(B_Q_FULL), q_phase, ab, 25))) {
          ok = false;
          break;
        }
        const uint32_t qrow = base + OFF_Q + (uint32_t)t * kTileBytes + (uint32_t)tid * 128u;
#pragma unroll 1
        for (int c = 0; c < 16; ++c) {  // 16-byte chunks: box c / 8, chunk c % 8
          const uint32_t a = qrow + (uint32_t)(c >> 3) * kBoxBytes +
                             ((((uint32_t)c & 7u) ^ ((uint32_t)tid & 7u)) << 4);
          uint32_t w[4];
          asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]) : "r"(a));
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            float cs, sn;
            rope_cos_sin_fast(row, freq[4 * c + u], &cs, &sn);
            const float x0 = __uint_as_float(w[u] << 16), x1 = __uint_as_float(w[u] & 0xffff0000u);
            w[u] = pack_bf16(x0 * cs - x1 * sn, x0 * sn + x1 * cs);
          }
          st_shared_v4(a, w[0], w[1], w[2], w[3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_Q_ROT + t));
      }
      const bool row_ok = row < p.S;
      int32_t seg_row = row_ok ? (p.seg ? p.seg[(size_t)it.b * p.S + row] : 0) : -1;
      const size_t tok = (size_t)it.b * p.S + (size_t)(row_ok ? row : 0);
      float m = -INFINITY, l = 0.f;
      int ntiles = 0;
      for (int j = lo_t; j <= hi_t; ++j) {
        // tile needs element masking?
        bool partial = (p.causal && j == qt_t) || ((int64_t)(j + 1) * 128 > p.S);
        if (p.seg) {
          const size_t kj = (size_t)it.b * p.n_tiles + j;
          const int32_t a0 = p.ktmin[kj], a1 = p.ktmax[kj];
          if (!meet(qmin_t, qmax_t, a0, a1)) continue;  // no query meets a key of tile j
          partial |= !(qmin_t >= 0 && qmin_t == qmax_t && a0 == qmin_t && a1 == qmin_t);
        }
        // packing: lane c's key segment ids (columns 32w + c), loaded before
        // the wait for S so that their latency overlaps it
        const int64_t kvalid = p.S - (int64_t)j * 128;
        int32_t kseg[4] = {INT_MIN, INT_MIN, INT_MIN, INT_MIN};
        if (partial && p.seg) {
          const int32_t* ks = p.kseg + (size_t)it.b * p.S + (size_t)j * 128;
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            const int64_t kc = 32 * w + lane;
            if (kc < kvalid) kseg[w] = __ldg(ks + kc);
          }
        }
        // every thread of the warp must agree before the .sync.aligned TMEM ops
        if (!__all_sync(0xffffffffu, mbar_wait(bar(B_S_FULL + t), s_cnt & 1, ab, 10 + t))) {
          ok = false;
          break;
        }
        ++s_cnt;
        tc_fence_after();
        // S row in registers (raw scores); masked entries become -inf.
        uint32_t r[128];
#pragma unroll
        for (int c = 0; c < 4; ++c)
          tmem_ld32(tS + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&r[c * 32]));
        tmem_wait_ld();
        if (partial) {
          // keys c <= lim are inside the row's causal window and the sequence
          const int64_t d = row - (int64_t)j * 128;
          int lim = p.causal ? (int)(d < -1 ? -1 : (d > 127 ? 127 : d)) : 127;
          if (kvalid - 1 < lim) lim = (int)(kvalid - 1);
          if (seg_row < 0) lim = -1;
          // 128-bit keep mask, built without touching the score registers:
          // keys 32w + c <= lim, and (packing) the row's segment
          uint32_t mw[4];
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            const int n = lim - 32 * w + 1;
            uint32_t bits = bit_range(0, n < 0 ? 0 : (n > 32 ? 32 : n));
            if (p.seg) bits &= warp_segment_bits(kseg[w], seg_row);
            mw[w] = bits;
          }
#pragma unroll
          for (int c = 0; c < 128; ++c)
            r[c] = ((mw[c >> 5] >> (c & 31)) & 1u) ? r[c] : 0xff800000u;
        }
        float mxr = -INFINITY;
#pragma unroll
        for (int c = 0; c < 128; ++c) mxr = fmaxf(mxr, __uint_as_float(r[c]));
        const float mx = mxr * p.scale_log2;  // scale > 0 keeps the order
        float fscale = 1.f;  // factor for O when the running max moves
        if (mx != -INFINITY) {
          if (m == -INFINITY) {
            m = mx;
          } else if (mx > m + kRescaleLog2) {
            fscale = fast_exp2(m - mx);
            l *= fscale;
            m = mx;
          }
        }
        const float neg_m = (m == -INFINITY) ? 0.f : -m;
        float sum = 0.f;
        // p = 2^(s * scale * log2e - m), packed two bf16 per column in place
#pragma unroll
        for (int u = 0; u < 64; ++u) {
          const float p0 = fast_exp2(fmaf(__uint_as_float(r[2 * u]), p.scale_log2, neg_m));
          const float p1 = fast_exp2(fmaf(__uint_as_float(r[2 * u + 1]), p.scale_log2, neg_m));
          sum += p0 + p1;
          r[u] = pack_bf16(p0, p1);
        }
        tmem_st32(tS, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
        tmem_st32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
        if (__any_sync(0xffffffffu, fscale != 1.f)) {  // warp-uniform: TMEM ops are .sync.aligned
          // the previous PV of this tile has completed (it was issued before
          // the S MMA whose completion this thread waited for)
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t o[32];
            tmem_ld32(tO + c * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int u = 0; u < 32; ++u) o[u] = __float_as_uint(__uint_as_float(o[u]) * fscale);
            tmem_st32(tO + c * 32, o);
          }
        }
        l += sum;
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(B_P_FULL + t));
        ++ntiles;
      }
      if (!ok) break;
      __nv_bfloat16* orow = p.o + (tok * p.H + it.h) * kD;
      float* orow32 = p.o32 + (tok * p.H + it.h) * kD;
      if (ntiles == 0) {
        if (row_ok) {
          const uint4 z = make_uint4(0, 0, 0, 0);
          if (p.o32) {
#pragma unroll
            for (int c = 0; c < 32; ++c) reinterpret_cast<uint4*>(orow32)[c] = z;
          } else {
#pragma unroll
            for (int c = 0; c < 16; ++c) reinterpret_cast<uint4*>(orow)[c] = z;
          }
          p.lse[((size_t)it.b * p.H + it.h) * p.S + row] = -INFINITY;
        }
        continue;
      }
      if (!__all_sync(0xffffffffu, mbar_wait(bar(B_O_FULL + t), o_cnt & 1, ab, 12 + t))) {
        ok = false;
        break;
      }
      ++o_cnt;
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      if (p.o32) {
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t r[32];
          tmem_ld32(tO + c * 32, r);
          tmem_wait_ld();
          if (!row_ok) continue;
          float4* dst = reinterpret_cast<float4*>(orow32 + c * 32);
#pragma unroll
          for (int u = 0; u < 8; ++u)
            dst[u] = make_float4(__uint_as_float(r[4 * u]) * inv, __uint_as_float(r[4 * u + 1]) * inv,
                                 __uint_as_float(r[4 * u + 2]) * inv, __uint_as_float(r[4 * u + 3]) * inv);
        }
      } else {
        // bf16 O through this warp's 2 KB of shared memory, 32 columns at a
        // time: each lane writes its row's four 16-byte chunks, then each
        // store instruction covers 8 rows x 64 contiguous bytes instead of 32
        // rows x 16 bytes.  Chunk ch of row r sits at slot ch ^ ((r >> 1) & 3),
        // which keeps both the row-wise writes and the column-wise reads free
        // of bank conflicts.
        const uint32_t stg = base + OFF_STG + (uint32_t)(warp - 4) * kStgWarpBytes;
        const int rr = lane & 7, cc = lane >> 3;  // read side: rows 8k + rr, chunk cc
        const int64_t row0 = (int64_t)qt_t * 128 + 32 * (warp & 3);  // this warp's first row
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t r[32];
          tmem_ld32(tO + c * 32, r);
          tmem_wait_ld();
          uint32_t pk[16];
#pragma unroll
          for (int u = 0; u < 16; ++u)
            pk[u] = pack_bf16(__uint_as_float(r[2 * u]) * inv, __uint_as_float(r[2 * u + 1]) * inv);
#pragma unroll
          for (int ch = 0; ch < 4; ++ch)
            st_shared_v4(stg + (uint32_t)lane * 64u + (uint32_t)((ch ^ ((lane >> 1) & 3)) << 4),
                         pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
          __syncwarp();
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int rw = 8 * k + rr;  // row within this warp's 32
            uint32_t v[4];
            asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3])
                         : "r"(stg + (uint32_t)rw * 64u + (uint32_t)((cc ^ ((rw >> 1) & 3)) << 4)));
            const int64_t orow_k = row0 + rw;
            if (orow_k < p.S) {
              __nv_bfloat16* dst =
                  p.o + (((size_t)it.b * p.S + (size_t)orow_k) * p.H + it.h) * kD + c * 32 + cc * 8;
              *reinterpret_cast<uint4*>(dst) = make_uint4(v[0], v[1], v[2], v[3]);
            }
          }
          __syncwarp();
        }
      }
      if (row_ok)
        p.lse[((size_t)it.b * p.H + it.h) * p.S + row] =
            l > 0.f ? (m + __log2f(l)) * 0.6931471805599453f : -INFINITY;
      tc_fence_before();
      mbar_arrive(bar(B_O_EMPTY + t));
    }
  }

  // ------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    if (warp == 1 && lane == 0) {
      mma_commit(bar(B_FIN));
      drain_wait(bar(B_FIN), 0);
    }
    if (warp == 0 && lane == 0) {
      // at most one load in flight per ring stage: the latest one issued
      for (uint32_t n = (k_issued > 2 ? k_issued - 2 : 0); n < k_issued; ++n)
        drain_wait(bar(B_K_FULL + (n & 1)), (n >> 1) & 1);
      for (uint32_t n = (v_issued > 2 ? v_issued - 2 : 0); n < v_issued; ++n)
        drain_wait(bar(B_V_FULL + (n & 1)), (n >> 1) & 1);
    }
  }
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

}  // namespace

// [B, S, H, D] bf16 as a 4-D tensor map {D, H, S, B}, 64 x 1 x box_rows x 1
// boxes, 128-byte swizzle (the canonical K-major / MN-major SW128 operand
// layout).
bool make_bf16_map(CUtensorMap* map, const void* ptr, int64_t B, int64_t S, int64_t H, int64_t D,
                   int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)S, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)(D * 2), (cuuint64_t)(H * D * 2), (cuuint64_t)(S * H * D * 2)};
  cuuint32_t box[4] = {64, 1, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_qkv_map(CUtensorMap* map, const void* ptr, int64_t B, int64_t S, int64_t H, int64_t D) {
  return make_bf16_map(map, ptr, B, S, H, D, 128);
}

// [B, S, H, D] bf16 tensor written by 32-row x 32-column boxes (64-byte
// rows) from shared memory in the 64-byte swizzle: the store map of the
// one-pass backward's dK / dV epilogue.
bool make_bf16_store_map(CUtensorMap* map, const void* ptr, int64_t B, int64_t S, int64_t H,
                         int64_t D) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)S, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)(D * 2), (cuuint64_t)(H * D * 2), (cuuint64_t)(S * H * D * 2)};
  cuuint32_t box[4] = {32, 1, 32, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                  CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int sm_count() {
  int dev = 0, n = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

bool sm100_available() {
  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  return major == 10 && minor == 0 && encode_fn() != nullptr;
}

cudaError_t launch_sm100_fwd(const Problem& pb, const Workspace& ws, const void* q, const void* v,
                             void* o, float* lse, cudaStream_t st, bool o_f32) {
  CUtensorMap tq, tk, tv;
  const bool rot_q = rope_on_load_fwd(pb);  // else the workspace holds the rotated q
  if (!make_qkv_map(&tq, rot_q ? q : ws.q_rot, pb.B, pb.S, pb.H, pb.D) ||
      !make_qkv_map(&tk, ws.k_rot, pb.B, pb.S, pb.H, pb.D) ||
      !make_qkv_map(&tv, v, pb.B, pb.S, pb.H, pb.D))
    return cudaErrorInvalidValue;
  FwdParams p{};
  p.seg = pb.seg;
  p.kseg = pb.kseg;
  p.tmin = ws.tile_min;
  p.tmax = ws.tile_max;
  p.ktmin = ws.ktile_min;
  p.ktmax = ws.ktile_max;
  p.q_lo = ws.q_lo;
  p.o = o_f32 ? nullptr : static_cast<__nv_bfloat16*>(o);
  p.o32 = o_f32 ? static_cast<float*>(o) : nullptr;
  p.lse = lse;
  p.status = ws.status;
  p.S = pb.S;
  p.H = (int)pb.H;
  p.B = (int)pb.B;
  p.n_tiles = (int)pb.n_tiles;
  p.n_pairs = (int)((pb.n_tiles + 1) / 2);
  p.scale_log2 = pb.scale * 1.4426950408889634f;
  p.causal = pb.causal;
  p.rotate = rot_q;
  p.log2_theta = p.rotate ? log2(pb.theta) : 0.0;
  const int64_t n_items = pb.B * pb.H * p.n_pairs;
  if (n_items == 0) return cudaSuccess;
  static std::once_flag attr_once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(attr_once, [] {
    attr_err = cudaFuncSetAttribute(attn_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)kSmemBytes);
  });
  if (attr_err != cudaSuccess) return attr_err;
  const int grid = (int)(n_items < sm_count() ? n_items : sm_count());
  attn_fwd_kernel<<<grid, kThreads, kSmemBytes, st>>>(tq, tk, tv, p);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace lwm
