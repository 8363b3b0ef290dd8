// Forward attention for fp32 inputs on the 5th-generation tensor cores
// (sm_100a), head_dim 64 or 128.
//
// The pages train and infer in fp32 (LWM research note, "Infra"); the bf16
// tensor cores reach fp32-level accuracy here through split operands.  Each
// fp32 operand x is carried as two bf16 planes, hi = bf16(x) and lo =
// bf16(x - hi) (together about 16 significant bits), and every product is
// the sum of three bf16 products accumulated in fp32 tensor memory:
//   x * y  ~  hi(x) hi(y) + hi(x) lo(y) + lo(x) hi(y)
// (the dropped lo * lo term is below 2^-16 relative).  The split pre-pass
// applies RoPE in fp32 first.  P is split the same way before the PV
// product.  What it computes is the forward of the tensor-core bf16 path
// (exact causal softmax attention with a packing mask), O and LSE in fp32.
//
// Design (one persistent CTA per SM, 192 threads):
//   warp 0      TMA producer: per 64-key step the hi and lo planes of K~ and
//               of V through 3-stage rings (K runs two steps ahead of V).
//   warp 1      MMA issuer (one thread); the whole warp allocates and frees
//               the tensor memory.
//   warps 2-5   softmax, one query row per thread: Q~ hi/lo rows into tensor
//               memory at the start of an item, then per step S from TMEM,
//               mask, online max/sum (exp2, max kept stale until the true one
//               is 2^8 larger), P split into hi/lo bf16 over S, and the
//               epilogue (O/l in fp32, LSE).
// TMEM columns (D = 128; D = 64 halves the D-wide regions):
//   Q~hi [0,64) Q~lo [64,128) (bf16 pairs, A of S), S0 [128,192),
//   S1 [192,256) (64 keys each; P hi/lo over them, A of PV), Oa [256,384),
//   Ob [384,512).
// S is double-buffered and PV alternates between the two O accumulators, so
// the MMA of step j+1's scores and step j's PV run while the softmax works,
// and a rescale of O (when the running max moves) always touches the
// accumulator that no PV in flight is writing; the other one carries its
// pending factor until its own turn.  O = (Oa fa + Ob fb) / l at the end.
// MMA issue order: S(0) S(1) | PV(0) S(2) | PV(1) S(3) | ...
#include <cuda.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace lwm {

bool make_bf16_map(CUtensorMap* map, const void* ptr, int64_t B, int64_t S, int64_t H, int64_t D,
                   int box_rows);
int sm_count();

namespace {

using namespace sm100;

constexpr int kThreads = 192;
constexpr int kKeys = 64;                 // keys per step
constexpr uint32_t kBox = 64 * 64 * 2;    // one TMA box: 64 columns x 64 rows of bf16
constexpr float kRescaleLog2 = 8.0f;
constexpr int kStages = 3;

template <int D> struct X3Cfg {
  static constexpr uint32_t kPlane = kBox * (D / 64);   // one plane of a 64-key tile
  static constexpr uint32_t kStage = 2 * kPlane;        // hi + lo
  static constexpr uint32_t OFF_K = 0;
  static constexpr uint32_t OFF_V = OFF_K + kStages * kStage;
  static constexpr uint32_t OFF_SMALL = OFF_V + kStages * kStage;
  static constexpr uint32_t kSmemBytes = OFF_SMALL + 256 + 64 + 1024;
  // TMEM columns
  static constexpr uint32_t T_QHI = 0, T_QLO = D / 2, T_S0 = D, T_S1 = D + 64, T_OA = D + 128,
                            T_OB = 2 * D + 128;
};

enum : uint32_t {
  B_K_FULL = 0,    // kStages
  B_K_EMPTY = 3,
  B_V_FULL = 6,
  B_V_EMPTY = 9,
  B_Q_READY = 12,
  B_S_FULL = 13,   // per S buffer: each completes once per use of its buffer,
  B_P_FULL = 15,   // so a waiter is never more than one phase behind
  B_O_FULL = 17, B_FIN = 18,
  B_ITEM_FULL = 19,   // 4 slots
  B_ITEM_EMPTY = 23,  // 4 slots
  B_COUNT = 27
};
static_assert(B_COUNT * 8 <= 256, "barrier slots");
constexpr uint32_t kItemSlots = 4;
constexpr uint32_t kSoftmaxWarps = 4;

struct X3Params {
  const int32_t* seg;    // [B, S] query segment ids, or null
  const int32_t* kseg;   // key segment ids (seg unless a block pair)
  const int32_t* tmin;   // [B, nT] query tile bounds (128-row tiles)
  const int32_t* tmax;
  const int32_t* ktmin;  // key tile bounds
  const int32_t* ktmax;
  const int32_t* q_lo;   // first 128-key tile a query tile may need
  const __nv_bfloat16* q_hi;  // [B, S, H, D] planes of the rotated q
  const __nv_bfloat16* q_lo_plane;
  float* o;              // [B, S, H, D] fp32
  float* lse;            // [B, H, S]
  DeviceStatus* status;
  int64_t S;
  int H, B, n_tiles, n_k64;
  float scale_log2;
  int causal;
};

struct Item {
  int b, h, qt;
  int lo, hi;            // 64-key block range
  int32_t qmin, qmax;
};

__device__ __forceinline__ bool meet(int32_t a0, int32_t a1, int32_t b0, int32_t b1) {
  return a1 >= 0 && b1 >= 0 && a0 <= b1 && b0 <= a1;
}

__device__ __forceinline__ Item decode(const X3Params& p, int idx) {
  Item it;
  const int bh = idx / p.n_tiles;
  it.qt = p.n_tiles - 1 - (idx % p.n_tiles);  // most key blocks first (causal)
  it.b = bh / p.H;
  it.h = bh % p.H;
  it.lo = 0;
  it.hi = p.causal ? min(2 * it.qt + 1, p.n_k64 - 1) : p.n_k64 - 1;
  it.qmin = 0;
  it.qmax = 0;
  if (p.seg) {
    const size_t ti = (size_t)it.b * p.n_tiles + it.qt;
    it.lo = 2 * p.q_lo[ti];
    it.qmin = p.tmin[ti];
    it.qmax = p.tmax[ti];
  }
  return it;
}

__device__ __forceinline__ bool rel(const X3Params& p, const Item& it, int kb) {
  if (kb < it.lo || kb > it.hi) return false;
  if (!p.seg) return true;
  const size_t kt = (size_t)it.b * p.n_tiles + (kb >> 1);
  return meet(it.qmin, it.qmax, p.ktmin[kt], p.ktmax[kt]);
}

__device__ __forceinline__ int next_rel(const X3Params& p, const Item& it, int kb) {
  for (++kb; kb <= it.hi; ++kb)
    if (rel(p, it, kb)) return kb;
  return -1;
}

__device__ __forceinline__ int first_rel(const X3Params& p, const Item& it) {
  if (it.lo > it.hi) return -1;
  return rel(p, it, it.lo) ? it.lo : next_rel(p, it, it.lo);
}

__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try(bar, parity)) {
    if (clock64() - t0 > kWaitCycles) return;
  }
}

// S (+)= A * B^T: A (bf16 pairs) in TMEM from column a_col, D/16 k-steps of
// 8 columns; B a 64-row K-major plane of 64-column boxes (kBox bytes each).
template <int D>
__device__ __forceinline__ void mma_s_part(uint32_t d, uint32_t a_col, uint64_t b_desc,
                                           uint32_t idesc, uint32_t acc) {
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint64_t off = (uint64_t)(((kk >> 2) * kBox + (kk & 3) * 32) >> 4);
    mma_ts(d, a_col + (uint32_t)(kk * 8), b_desc + off, idesc, kk > 0 ? 1u : acc);
  }
}

// O (+)= P * V over 64 keys: P (bf16 pairs) in TMEM from column a_col (4
// k-steps of 8 columns), V a 64-row MN-major plane (rows = keys).
__device__ __forceinline__ void mma_pv_part(uint32_t d, uint32_t a_col, uint64_t b_desc,
                                            uint32_t idesc, uint32_t acc) {
#pragma unroll
  for (int kk = 0; kk < 4; ++kk)
    mma_ts(d, a_col + (uint32_t)(kk * 8), b_desc + (uint64_t)((kk * 2048) >> 4), idesc,
           kk > 0 ? 1u : acc);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
attn_fwd_x3_kernel(const __grid_constant__ CUtensorMap tm_khi, const __grid_constant__ CUtensorMap tm_klo,
                   const __grid_constant__ CUtensorMap tm_vhi, const __grid_constant__ CUtensorMap tm_vlo,
                   const X3Params p) {
  using C = X3Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  const uint32_t bar0 = base + C::OFF_SMALL;
  auto bar = [&](uint32_t slot) { return bar0 + 8u * slot; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_SMALL + 256 + 8);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_SMALL + 256);
  volatile int* item_slot = reinterpret_cast<volatile int*>(smem + C::OFF_SMALL + 256 + 16);
  int* item_counter = &p.status->item_counter[2];
  const Abort ab{abort_flag, p.status};
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_items = p.B * p.H * p.n_tiles;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(B_K_FULL + s), 1);
      mbar_init(bar(B_K_EMPTY + s), 1);
      mbar_init(bar(B_V_FULL + s), 1);
      mbar_init(bar(B_V_EMPTY + s), 1);
    }
    mbar_init(bar(B_Q_READY), kSoftmaxWarps);
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(B_S_FULL + b), 1);
      mbar_init(bar(B_P_FULL + b), kSoftmaxWarps);
    }
    mbar_init(bar(B_O_FULL), 1);
    mbar_init(bar(B_FIN), 1);
    for (uint32_t sl = 0; sl < kItemSlots; ++sl) {
      mbar_init(bar(B_ITEM_FULL + sl), 1);
      mbar_init(bar(B_ITEM_EMPTY + sl), 1 + kSoftmaxWarps);
    }
    fence_mbar_init();
    tma_prefetch_desc(&tm_khi);
    tma_prefetch_desc(&tm_klo);
    tma_prefetch_desc(&tm_vhi);
    tma_prefetch_desc(&tm_vlo);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  uint32_t k_issued = 0, v_issued = 0;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA
    if (lane == 0) {
      uint32_t k_it = 0, v_it = 0;
      bool ok = true;
      for (uint32_t pub = 0; ok;) {
        const uint32_t sl = pub % kItemSlots;
        if (pub >= kItemSlots &&
            !mbar_wait(bar(B_ITEM_EMPTY + sl), ((pub / kItemSlots) - 1) & 1, ab, 110)) {
          ok = false;
          break;
        }
        const int idx = atomicAdd(item_counter, 1);
        item_slot[sl] = idx;
        mbar_arrive(bar(B_ITEM_FULL + sl));
        ++pub;
        if (idx >= n_items) break;
        const Item it = decode(p, idx);
        auto load = [&](bool is_k, int kb) -> bool {
          uint32_t& cnt = is_k ? k_it : v_it;
          const uint32_t s = cnt % kStages, n = cnt / kStages;
          const uint32_t full = bar((is_k ? B_K_FULL : B_V_FULL) + s);
          if (!mbar_wait(bar((is_k ? B_K_EMPTY : B_V_EMPTY) + s), (n & 1) ^ 1, ab, is_k ? 111 : 112))
            return false;
          mbar_expect_tx(full, C::kStage);
          const uint32_t dst = base + (is_k ? C::OFF_K : C::OFF_V) + s * C::kStage;
          const CUtensorMap* mh = is_k ? &tm_khi : &tm_vhi;
          const CUtensorMap* ml = is_k ? &tm_klo : &tm_vlo;
#pragma unroll
          for (int bx = 0; bx < D / 64; ++bx) {
            tma_load_4d(dst + bx * kBox, mh, full, 64 * bx, it.h, kb * kKeys, it.b);
            tma_load_4d(dst + C::kPlane + bx * kBox, ml, full, 64 * bx, it.h, kb * kKeys, it.b);
          }
          ++cnt;
          if (is_k) k_issued = cnt; else v_issued = cnt;
          return true;
        };
        // K runs two steps ahead of V (S(j+2) is issued right after PV(j))
        int kk = first_rel(p, it);
        for (int a = 0; a < 2 && kk >= 0 && ok; ++a, kk = next_rel(p, it, kk)) ok = load(true, kk);
        for (int kv = first_rel(p, it); kv >= 0 && ok; kv = next_rel(p, it, kv)) {
          ok = load(false, kv);
          if (ok && kk >= 0) {
            ok = load(true, kk);
            kk = next_rel(p, it, kk);
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA
    if (lane == 0) {
      constexpr uint32_t kIdS = idesc_bf16(128, kKeys, 0, 0);   // Q (TMEM) x K (K-major)
      constexpr uint32_t kIdPV = idesc_bf16(128, D, 0, 1);      // P (TMEM) x V (MN-major)
      uint32_t k_it = 0, v_it = 0, qrc = 0, p_use[2] = {0, 0};
      bool ok = true;
      auto kstage = [&](uint32_t n) { return base + C::OFF_K + (n % kStages) * C::kStage; };
      auto vstage = [&](uint32_t n) { return base + C::OFF_V + (n % kStages) * C::kStage; };
      auto issue_s = [&](uint32_t buf) -> bool {
        if (!mbar_wait(bar(B_K_FULL + k_it % kStages), (k_it / kStages) & 1, ab, 113)) return false;
        tc_fence_after();
        const uint32_t d = tmem + (buf ? C::T_S1 : C::T_S0);
        const uint64_t bh = kmajor_desc(kstage(k_it)), bl = kmajor_desc(kstage(k_it) + C::kPlane);
        mma_s_part<D>(d, tmem + C::T_QHI, bh, kIdS, 0u);
        mma_s_part<D>(d, tmem + C::T_QHI, bl, kIdS, 1u);
        mma_s_part<D>(d, tmem + C::T_QLO, bh, kIdS, 1u);
        mma_commit(bar(B_S_FULL + buf));
        mma_commit(bar(B_K_EMPTY + k_it % kStages));
        ++k_it;
        return true;
      };
      for (uint32_t cons = 0; ok;) {
        const uint32_t sl = cons % kItemSlots;
        if (!mbar_wait(bar(B_ITEM_FULL + sl), (cons / kItemSlots) & 1, ab, 114)) { ok = false; break; }
        const int idx = item_slot[sl];
        mbar_arrive(bar(B_ITEM_EMPTY + sl));
        ++cons;
        if (idx >= n_items) break;
        const Item it = decode(p, idx);
        int kb = first_rel(p, it);
        if (kb < 0) continue;
        // Q~ hi/lo rows in TMEM (the softmax warps wrote them after reading
        // out the previous item's O)
        if (!mbar_wait(bar(B_Q_READY), qrc & 1, ab, 115)) { ok = false; break; }
        ++qrc;
        int n = 0;
        for (int t = kb; t >= 0; t = next_rel(p, it, t)) ++n;
        if (!issue_s(0)) { ok = false; break; }
        if (n > 1 && !issue_s(1)) { ok = false; break; }
        for (int j = 0; j < n && ok; ++j) {
          if (!mbar_wait(bar(B_P_FULL + (j & 1)), p_use[j & 1] & 1, ab, 116)) { ok = false; break; }
          ++p_use[j & 1];
          if (!mbar_wait(bar(B_V_FULL + v_it % kStages), (v_it / kStages) & 1, ab, 117)) { ok = false; break; }
          tc_fence_after();
          const uint32_t s = tmem + ((j & 1) ? C::T_S1 : C::T_S0);
          const uint32_t d = tmem + ((j & 1) ? C::T_OB : C::T_OA);
          const uint64_t bh = mnmajor_desc_lbo(vstage(v_it), kBox);
          const uint64_t bl = mnmajor_desc_lbo(vstage(v_it) + C::kPlane, kBox);
          mma_pv_part(d, s, bh, kIdPV, j >= 2 ? 1u : 0u);       // P hi x V hi
          mma_pv_part(d, s, bl, kIdPV, 1u);                     // P hi x V lo
          mma_pv_part(d, s + 32u, bh, kIdPV, 1u);               // P lo x V hi
          mma_commit(bar(B_V_EMPTY + v_it % kStages));
          ++v_it;
          if (j + 2 < n && !issue_s(j & 1)) { ok = false; break; }
        }
        if (!ok) break;
        mma_commit(bar(B_O_FULL));
      }
    }
  } else {
    // -------------------------------------------------------------- softmax
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // TMEM lane = row in the query tile
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    uint32_t s_use[2] = {0, 0}, o_cnt = 0;
    bool ok = true;
    for (uint32_t cons = 0; ok;) {
      const uint32_t sl = cons % kItemSlots;
      if (!__all_sync(0xffffffffu, mbar_wait(bar(B_ITEM_FULL + sl), (cons / kItemSlots) & 1, ab, 118))) {
        ok = false;
        break;
      }
      const int idx = item_slot[sl];
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_ITEM_EMPTY + sl));
      ++cons;
      if (idx >= n_items) break;
      const Item it = decode(p, idx);
      const int64_t row = (int64_t)it.qt * 128 + r;
      const bool row_ok = row < p.S;
      const int32_t seg_row = row_ok ? (p.seg ? p.seg[(size_t)it.b * p.S + row] : 0) : -1;
      const size_t tok = (size_t)it.b * p.S + (size_t)(row_ok ? row : 0);
      float* orow = p.o + (tok * p.H + it.h) * D;
      const int kb0 = first_rel(p, it);
      if (kb0 < 0) {
        if (row_ok) {
          const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
          for (int c = 0; c < D / 4; ++c) reinterpret_cast<float4*>(orow)[c] = z;
          p.lse[((size_t)it.b * p.H + it.h) * p.S + row] = -INFINITY;
        }
        continue;
      }
      // this row of Q~ hi and lo into TMEM (zeros past the end)
      {
        const size_t off = (tok * p.H + it.h) * D;
        const uint4* qh = reinterpret_cast<const uint4*>(p.q_hi + off);
        const uint4* ql = reinterpret_cast<const uint4*>(p.q_lo_plane + off);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const uint4* src = half ? ql : qh;
#pragma unroll
          for (int c0 = 0; c0 < D / 64; ++c0) {   // 32 columns = 64 values per store
            uint32_t v[32];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const uint4 a = row_ok ? src[c0 * 8 + u] : make_uint4(0, 0, 0, 0);
              v[4 * u] = a.x; v[4 * u + 1] = a.y; v[4 * u + 2] = a.z; v[4 * u + 3] = a.w;
            }
            tmem_st32(tmem + lane_base + (half ? C::T_QLO : C::T_QHI) + 32u * c0, v);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_Q_READY));
      }
      float m = -INFINITY, l = 0.f, pend[2] = {1.f, 1.f};
      int j = 0;
      for (int kb = kb0; kb >= 0; kb = next_rel(p, it, kb), ++j) {
        const int64_t k0 = (int64_t)kb * kKeys;
        bool partial = (p.causal && k0 + kKeys - 1 > (int64_t)it.qt * 128) || (k0 + kKeys > p.S);
        if (p.seg) {
          const size_t kt = (size_t)it.b * p.n_tiles + (kb >> 1);
          const int32_t a0 = p.ktmin[kt], a1 = p.ktmax[kt];
          partial |= !(it.qmin >= 0 && it.qmin == it.qmax && a0 == it.qmin && a1 == it.qmin);
        }
        if (!__all_sync(0xffffffffu, mbar_wait(bar(B_S_FULL + (j & 1)), s_use[j & 1] & 1, ab, 119))) {
          ok = false;
          break;
        }
        ++s_use[j & 1];
        tc_fence_after();
        const uint32_t tS = tmem + lane_base + ((j & 1) ? C::T_S1 : C::T_S0);
        uint32_t sr[64];
        tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
        tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
        tmem_wait_ld();
        if (partial) {
          const int64_t d = row - k0;
          const int64_t kvalid = p.S - k0;
          int lim = p.causal ? (int)(d < -1 ? -1 : (d > 63 ? 63 : d)) : 63;
          if (kvalid - 1 < lim) lim = (int)(kvalid - 1);
          if (seg_row < 0) lim = -1;
          const int32_t* ks = p.seg ? p.kseg + (size_t)it.b * p.S + (size_t)k0 : nullptr;
          uint32_t mw[2];
#pragma unroll
          for (int g = 0; g < 2; ++g) {
            const int nb = lim - 32 * g + 1;
            uint32_t bits = bit_range(0, nb < 0 ? 0 : (nb > 32 ? 32 : nb));
            if (ks) {
              const int64_t kc = 32 * g + lane;
              const int32_t kseg = kc < kvalid ? __ldg(ks + kc) : INT_MIN;
              bits &= warp_segment_bits(kseg, seg_row);
            }
            mw[g] = bits;
          }
#pragma unroll
          for (int c = 0; c < 64; ++c)
            sr[c] = ((mw[c >> 5] >> (c & 31)) & 1u) ? sr[c] : 0xff800000u;
        }
        float mxr = -INFINITY;
#pragma unroll
        for (int c = 0; c < 64; ++c) mxr = fmaxf(mxr, __uint_as_float(sr[c]));
        const float mx = mxr * p.scale_log2;
        float f = 1.f;  // factor for everything accumulated so far
        if (mx != -INFINITY) {
          if (m == -INFINITY) {
            m = mx;
          } else if (mx > m + kRescaleLog2) {
            f = exp2f(m - mx);
            m = mx;
          }
        }
        const float neg_m = (m == -INFINITY) ? 0.f : -m;
        float sum = 0.f;
        uint32_t ph[32], pl[32];
#pragma unroll
        for (int u = 0; u < 32; ++u) {
          const float p0 = fast_exp2(fmaf(__uint_as_float(sr[2 * u]), p.scale_log2, neg_m));
          const float p1 = fast_exp2(fmaf(__uint_as_float(sr[2 * u + 1]), p.scale_log2, neg_m));
          sum += p0 + p1;
          const uint32_t h = pack_bf16(p0, p1);
          ph[u] = h;
          pl[u] = pack_bf16(p0 - __uint_as_float(h << 16), p1 - __uint_as_float(h & 0xffff0000u));
        }
        tmem_st32(tS, ph);
        tmem_st32(tS + 32, pl);
        l = l * f + sum;
        // O accumulators: both hold contributions relative to the old max
        pend[0] *= f;
        pend[1] *= f;
        const int cur = j & 1;
        if (j < 2) {
          pend[cur] = 1.f;  // PV(j) starts this accumulator afresh
        } else if (__any_sync(0xffffffffu, pend[cur] != 1.f)) {
          // PV(j-2), the last writer of this accumulator, completed before
          // S(j) (issue order); PV(j) waits for P_FULL below
          const uint32_t tO = tmem + lane_base + (cur ? C::T_OB : C::T_OA);
          const float sc = pend[cur];
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(tO + c * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int u = 0; u < 32; ++u) o[u] = __float_as_uint(__uint_as_float(o[u]) * sc);
            tmem_st32(tO + c * 32, o);
          }
          pend[cur] = 1.f;
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_P_FULL + (j & 1)));
      }
      if (!ok) break;
      if (!__all_sync(0xffffffffu, mbar_wait(bar(B_O_FULL), o_cnt & 1, ab, 120))) {
        ok = false;
        break;
      }
      ++o_cnt;
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const float fa = pend[0] * inv, fb = (j >= 2 ? pend[1] : 0.f) * inv;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t oa[32], ob[32];
        tmem_ld32(tmem + lane_base + C::T_OA + c * 32, oa);
        tmem_ld32(tmem + lane_base + C::T_OB + c * 32, ob);
        tmem_wait_ld();
        if (row_ok) {
          float4* dst = reinterpret_cast<float4*>(orow + c * 32);
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            float x[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
              x[e] = __uint_as_float(oa[4 * u + e]) * fa +
                     (j >= 2 ? __uint_as_float(ob[4 * u + e]) * fb : 0.f);
            dst[u] = make_float4(x[0], x[1], x[2], x[3]);
          }
        }
      }
      if (row_ok)
        p.lse[((size_t)it.b * p.H + it.h) * p.S + row] =
            l > 0.f ? (m + __log2f(l)) * 0.6931471805599453f : -INFINITY;
      tc_fence_before();
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
      for (uint32_t n = (k_issued > kStages ? k_issued - kStages : 0); n < k_issued; ++n)
        drain_wait(bar(B_K_FULL + n % kStages), (n / kStages) & 1);
      for (uint32_t n = (v_issued > kStages ? v_issued - kStages : 0); n < v_issued; ++n)
        drain_wait(bar(B_V_FULL + n % kStages), (n / kStages) & 1);
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int D>
cudaError_t launch_x3(const Problem& pb, const Workspace& ws, float* o, float* lse, cudaStream_t st) {
  CUtensorMap khi, klo, vhi, vlo;
  if (!make_bf16_map(&khi, ws.kx_hi, pb.B, pb.S, pb.H, D, 64) ||
      !make_bf16_map(&klo, ws.kx_lo, pb.B, pb.S, pb.H, D, 64) ||
      !make_bf16_map(&vhi, ws.vx_hi, pb.B, pb.S, pb.H, D, 64) ||
      !make_bf16_map(&vlo, ws.vx_lo, pb.B, pb.S, pb.H, D, 64))
    return cudaErrorInvalidValue;
  X3Params p{};
  p.seg = pb.seg;
  p.kseg = pb.kseg;
  p.tmin = ws.tile_min;
  p.tmax = ws.tile_max;
  p.ktmin = ws.ktile_min;
  p.ktmax = ws.ktile_max;
  p.q_lo = ws.q_lo;
  p.q_hi = static_cast<const __nv_bfloat16*>(ws.qx_hi);
  p.q_lo_plane = static_cast<const __nv_bfloat16*>(ws.qx_lo);
  p.o = o;
  p.lse = lse;
  p.status = ws.status;
  p.S = pb.S;
  p.H = (int)pb.H;
  p.B = (int)pb.B;
  p.n_tiles = (int)pb.n_tiles;
  p.n_k64 = (int)((pb.S + kKeys - 1) / kKeys);
  p.scale_log2 = pb.scale * 1.4426950408889634f;
  p.causal = pb.causal;
  const int64_t n_items = pb.B * pb.H * pb.n_tiles;
  if (n_items == 0) return cudaSuccess;
  using C = X3Cfg<D>;
  static std::once_flag attr_once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(attr_once, [] {
    attr_err = cudaFuncSetAttribute(attn_fwd_x3_kernel<D>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::kSmemBytes);
  });
  if (attr_err != cudaSuccess) return attr_err;
  const int grid = (int)(n_items < sm_count() ? n_items : sm_count());
  attn_fwd_x3_kernel<D><<<grid, kThreads, C::kSmemBytes, st>>>(khi, klo, vhi, vlo, p);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_sm100_fwd_x3(const Problem& pb, const Workspace& ws, float* o, float* lse,
                                cudaStream_t st) {
  if (pb.D == 128) return launch_x3<128>(pb, ws, o, lse, st);
  if (pb.D == 64) return launch_x3<64>(pb, ws, o, lse, st);
  return cudaErrorInvalidValue;
}

}  // namespace lwm
