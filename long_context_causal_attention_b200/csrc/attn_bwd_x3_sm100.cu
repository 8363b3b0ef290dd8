// Backward attention for fp32 inputs on the 5th-generation tensor cores
// (sm_100a), head_dim 64 or 128, with split operands as in the fp32 forward
// (attn_fwd_x3_sm100.cu): every fp32 operand is a bf16 hi plane plus a bf16
// lo plane and every product is hi*hi + hi*lo + lo*hi accumulated in fp32
// tensor memory; P and dS are split in registers before they become MMA
// operands.  The gradients are those of the bf16 backward (FlashAttention
// recomputation of P from the saved LSE, D = dO . O), for training in fp32
// (LWM research note, "Infra").  Two kernels:
//
// attn_bwd_dq_x3_kernel  (query-stationary; one persistent CTA per SM, 320
//   threads) per query tile i, over 64-key blocks j:
//     S = Q~ K~_j^T, dP = dO V_j^T, dS = P o (dP - D), dQ~ += dS K~_j
//   warp 0 TMA (K~ and V hi/lo planes of a key block, 3-stage ring), warp 1
//   MMA issuer, warps 2-9 element-wise (lane quarter x 32-key half).
//   TMEM: Q~hi, Q~lo, dOhi, dOlo (A operands, D/2 columns each), S (64),
//   dP (64; dS hi/lo over it), dQ~ (D).
//   MMA order: S(0) dP(0) | S(1) once S(0) is read | dQ(0) after dS(0), dP(1)
//   | S(2) once S(1) is read | ...
//
// attn_bwd_dkdv_x3_kernel  (key-stationary; 320 threads) per key tile j,
//   over 64-query blocks i:
//     S^T = K~_j Q~_i^T, dP^T = V_j dO_i^T, dS^T = P^T o (dP^T - D_i),
//     dV_j += P^T dO_i, dK~_j += dS^T Q~_i
//   warp 0 TMA (K~ hi/lo once per item; Q~ and dO hi/lo planes of a query
//   block with its LSE*log2(e) and D, 2-stage ring), warp 1 MMA, warps 2-9
//   element-wise.  TMEM: Vhi, Vlo (A of dP^T, D/2 each), S^T (64; P^T hi/lo
//   over it), dP^T (64; dS^T hi/lo over it), dV (D), dK (D); K~ hi/lo as the
//   A operand of S^T in shared memory.
//   MMA order: S^T(0) dP^T(0) | dV(0) after P(0), S^T(1) | dK(0) after dS(0),
//   dP^T(1) | dV(1), S^T(2) | ...
// Epilogues scale dK~, dQ~ and undo the rotation (fp32 out).
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

constexpr int kThreads = 320;        // 2 control warps + 8 element-wise warps
constexpr int kEWWarps = 8;
constexpr uint32_t kBox64 = 64 * 64 * 2;    // TMA box: 64 columns x 64 rows of bf16
constexpr uint32_t kBox128 = 64 * 128 * 2;  // TMA box: 64 columns x 128 rows
constexpr uint32_t kItemSlots = 4;

__device__ __forceinline__ bool meet(int32_t a0, int32_t a1, int32_t b0, int32_t b1) {
  return a1 >= 0 && b1 >= 0 && a0 <= b1 && b0 <= a1;
}

__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try(bar, parity)) {
    if (clock64() - t0 > kWaitCycles) return;
  }
}

// (lo, hi) bf16 halves of a pair of floats, and the bf16 residuals
__device__ __forceinline__ void split_pair(float a, float b, uint32_t* hi, uint32_t* lo) {
  const uint32_t h = pack_bf16(a, b);
  *hi = h;
  *lo = pack_bf16(a - __uint_as_float(h << 16), b - __uint_as_float(h & 0xffff0000u));
}

// D (+)= A * B^T, A (bf16 pairs) in TMEM from a_col (D/16 k-steps of 8
// columns), B a 64-row K-major plane of 8 KB boxes.
template <int D>
__device__ __forceinline__ void mma_t_k64(uint32_t d, uint32_t a_col, uint64_t b_desc,
                                          uint32_t idesc, uint32_t acc) {
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk)
    mma_ts(d, a_col + (uint32_t)(kk * 8),
           b_desc + (uint64_t)(((kk >> 2) * kBox64 + (kk & 3) * 32) >> 4), idesc,
           kk > 0 ? 1u : acc);
}

// D (+)= A * B^T, A a 128-row K-major plane of 16 KB boxes in shared memory,
// B a 64-row K-major plane of 8 KB boxes.
template <int D>
__device__ __forceinline__ void mma_s128_k64(uint32_t d, uint64_t a_desc, uint64_t b_desc,
                                             uint32_t idesc, uint32_t acc) {
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk)
    mma_ss(d, a_desc + (uint64_t)(((kk >> 2) * kBox128 + (kk & 3) * 32) >> 4),
           b_desc + (uint64_t)(((kk >> 2) * kBox64 + (kk & 3) * 32) >> 4), idesc,
           kk > 0 ? 1u : acc);
}

// D (+)= A * B over 64 K rows: A (bf16 pairs) in TMEM from a_col (4 k-steps of
// 8 columns), B a 64-row MN-major plane (rows = K, 8 KB boxes along N).
__device__ __forceinline__ void mma_t_m64(uint32_t d, uint32_t a_col, uint64_t b_desc,
                                          uint32_t idesc, uint32_t acc) {
#pragma unroll
  for (int kk = 0; kk < 4; ++kk)
    mma_ts(d, a_col + (uint32_t)(kk * 8), b_desc + (uint64_t)((kk * 2048) >> 4), idesc,
           kk > 0 ? 1u : acc);
}

struct X3BwdParams {
  const int32_t* seg;
  const int32_t* kseg;
  const int32_t* tmin;
  const int32_t* tmax;
  const int32_t* ktmin;
  const int32_t* ktmax;
  const int32_t* q_lo;   // first 128-key tile a query tile may need
  const int32_t* k_hi;   // last 128-query tile a key tile may feed
  const float* lse2;     // [B, H, nT*128]
  const float* dpad;     // [B, H, nT*128]
  const __nv_bfloat16* a_hi;  // rows the element-wise warps put into TMEM:
  const __nv_bfloat16* a_lo;  //   Q~ (dQ kernel) or V (dK/dV kernel) planes
  const __nv_bfloat16* b_hi;  //   dO planes (dQ kernel only)
  const __nv_bfloat16* b_lo;
  float* out0;           // dq (dQ kernel) or dk (dK/dV kernel), fp32 [B, S, H, D]
  float* out1;           // dv (dK/dV kernel)
  DeviceStatus* status;
  int64_t S;
  int H, B, n_tiles, n_b64;
  float scale, scale_log2;
  int causal, rotate;
  double log2_theta;
};

// ============================================================== dQ kernel
template <int D> struct DqCfg {
  static constexpr uint32_t kPlane = kBox64 * (D / 64);  // 64 keys x D
  static constexpr uint32_t kStage = 4 * kPlane;         // K~ hi, lo, V hi, lo
  static constexpr int kStages = 3;
  static constexpr uint32_t OFF_SMALL = kStages * kStage;
  static constexpr uint32_t kSmemBytes = OFF_SMALL + 256 + 64 + (D / 2) * 8 + 1024;
  static constexpr uint32_t T_QHI = 0, T_QLO = D / 2, T_DOHI = D, T_DOLO = 3 * D / 2, T_S = 2 * D,
                            T_DP = 2 * D + 64, T_DQ = 2 * D + 128;
};

enum : uint32_t {
  Q_K_FULL = 0, Q_K_EMPTY = 3,   // 3 stages
  Q_A_READY = 6, Q_S_FULL = 7, Q_S_READ = 8, Q_DP_FULL = 9, Q_DS_FULL = 10, Q_DQ_FULL = 11,
  Q_FIN = 12, Q_ITEM_FULL = 13, Q_ITEM_EMPTY = 17, Q_COUNT = 21
};

struct DqItem {
  int b, h, i;
  int lo, hi;   // 64-key blocks
  int32_t qmin, qmax;
};

__device__ __forceinline__ DqItem dq_decode(const X3BwdParams& p, int idx) {
  DqItem it;
  const int bh = idx / p.n_tiles;
  it.i = p.n_tiles - 1 - (idx % p.n_tiles);
  it.b = bh / p.H;
  it.h = bh % p.H;
  it.lo = 0;
  it.hi = p.causal ? min(2 * it.i + 1, p.n_b64 - 1) : p.n_b64 - 1;
  it.qmin = 0;
  it.qmax = 0;
  if (p.seg) {
    const size_t ti = (size_t)it.b * p.n_tiles + it.i;
    it.lo = 2 * p.q_lo[ti];
    it.qmin = p.tmin[ti];
    it.qmax = p.tmax[ti];
  }
  return it;
}

__device__ __forceinline__ bool dq_rel(const X3BwdParams& p, const DqItem& it, int kb) {
  if (kb < it.lo || kb > it.hi) return false;
  if (!p.seg) return true;
  const size_t kt = (size_t)it.b * p.n_tiles + (kb >> 1);
  return meet(it.qmin, it.qmax, p.ktmin[kt], p.ktmax[kt]);
}

__device__ __forceinline__ int dq_next(const X3BwdParams& p, const DqItem& it, int kb) {
  for (++kb; kb <= it.hi; ++kb)
    if (dq_rel(p, it, kb)) return kb;
  return -1;
}

__device__ __forceinline__ int dq_first(const X3BwdParams& p, const DqItem& it) {
  if (it.lo > it.hi) return -1;
  return dq_rel(p, it, it.lo) ? it.lo : dq_next(p, it, it.lo);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
attn_bwd_dq_x3_kernel(const __grid_constant__ CUtensorMap tm_khi, const __grid_constant__ CUtensorMap tm_klo,
                      const __grid_constant__ CUtensorMap tm_vhi, const __grid_constant__ CUtensorMap tm_vlo,
                      const X3BwdParams p) {
  using C = DqCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  const uint32_t bar0 = base + C::OFF_SMALL;
  auto bar = [&](uint32_t slot) { return bar0 + 8u * slot; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_SMALL + 256 + 8);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_SMALL + 256);
  volatile int* item_slot = reinterpret_cast<volatile int*>(smem + C::OFF_SMALL + 256 + 16);
  double* freq = reinterpret_cast<double*>(smem + C::OFF_SMALL + 256 + 64);
  int* item_counter = &p.status->item_counter[1];
  const Abort ab{abort_flag, p.status};
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_items = p.B * p.H * p.n_tiles;
  constexpr int kSt = C::kStages;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int s = 0; s < kSt; ++s) {
      mbar_init(bar(Q_K_FULL + s), 1);
      mbar_init(bar(Q_K_EMPTY + s), 1);
    }
    mbar_init(bar(Q_A_READY), kEWWarps);
    mbar_init(bar(Q_S_FULL), 1);
    mbar_init(bar(Q_S_READ), kEWWarps);
    mbar_init(bar(Q_DP_FULL), 1);
    mbar_init(bar(Q_DS_FULL), kEWWarps);
    mbar_init(bar(Q_DQ_FULL), 1);
    mbar_init(bar(Q_FIN), 1);
    for (uint32_t sl = 0; sl < kItemSlots; ++sl) {
      mbar_init(bar(Q_ITEM_FULL + sl), 1);
      mbar_init(bar(Q_ITEM_EMPTY + sl), 1 + kEWWarps);
    }
    fence_mbar_init();
    tma_prefetch_desc(&tm_khi);
    tma_prefetch_desc(&tm_klo);
    tma_prefetch_desc(&tm_vhi);
    tma_prefetch_desc(&tm_vlo);
  }
  if (threadIdx.x >= 64 && threadIdx.x < 64 + D / 2 && p.rotate)
    freq[threadIdx.x - 64] = rope_freq(threadIdx.x - 64, D, p.log2_theta);
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  uint32_t k_issued = 0;

  if (warp == 0) {
    if (lane == 0) {
      uint32_t k_it = 0;
      bool ok = true;
      for (uint32_t pub = 0; ok;) {
        const uint32_t sl = pub % kItemSlots;
        if (pub >= kItemSlots &&
            !mbar_wait(bar(Q_ITEM_EMPTY + sl), ((pub / kItemSlots) - 1) & 1, ab, 130)) {
          ok = false;
          break;
        }
        const int idx = atomicAdd(item_counter, 1);
        item_slot[sl] = idx;
        mbar_arrive(bar(Q_ITEM_FULL + sl));
        ++pub;
        if (idx >= n_items) break;
        const DqItem it = dq_decode(p, idx);
        for (int kb = dq_first(p, it); kb >= 0 && ok; kb = dq_next(p, it, kb)) {
          const uint32_t s = k_it % kSt, n = k_it / kSt;
          if (!mbar_wait(bar(Q_K_EMPTY + s), (n & 1) ^ 1, ab, 131)) { ok = false; break; }
          const uint32_t full = bar(Q_K_FULL + s);
          mbar_expect_tx(full, C::kStage);
          const uint32_t dst = base + s * C::kStage;
#pragma unroll
          for (int bx = 0; bx < D / 64; ++bx) {
            tma_load_4d(dst + bx * kBox64, &tm_khi, full, 64 * bx, it.h, kb * 64, it.b);
            tma_load_4d(dst + C::kPlane + bx * kBox64, &tm_klo, full, 64 * bx, it.h, kb * 64, it.b);
            tma_load_4d(dst + 2 * C::kPlane + bx * kBox64, &tm_vhi, full, 64 * bx, it.h, kb * 64, it.b);
            tma_load_4d(dst + 3 * C::kPlane + bx * kBox64, &tm_vlo, full, 64 * bx, it.h, kb * 64, it.b);
          }
          k_issued = ++k_it;
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t kIdS = idesc_bf16(128, 64, 0, 0);   // TMEM x K-major, N = 64 keys
      constexpr uint32_t kIdQ = idesc_bf16(128, D, 0, 1);    // TMEM x MN-major, N = D
      uint32_t k_it = 0, arc = 0, s_read = 0, ds_full = 0;
      bool ok = true;
      auto stage = [&](uint32_t n) { return base + (n % kSt) * C::kStage; };
      auto wait_k = [&](uint32_t n) {
        return mbar_wait(bar(Q_K_FULL + n % kSt), (n / kSt) & 1, ab, 132);
      };
      auto issue_s = [&](uint32_t n) {
        const uint64_t bh = kmajor_desc(stage(n)), bl = kmajor_desc(stage(n) + C::kPlane);
        mma_t_k64<D>(tmem + C::T_S, tmem + C::T_QHI, bh, kIdS, 0u);
        mma_t_k64<D>(tmem + C::T_S, tmem + C::T_QHI, bl, kIdS, 1u);
        mma_t_k64<D>(tmem + C::T_S, tmem + C::T_QLO, bh, kIdS, 1u);
        mma_commit(bar(Q_S_FULL));
      };
      auto issue_dp = [&](uint32_t n) {
        const uint64_t vh = kmajor_desc(stage(n) + 2 * C::kPlane),
                       vl = kmajor_desc(stage(n) + 3 * C::kPlane);
        mma_t_k64<D>(tmem + C::T_DP, tmem + C::T_DOHI, vh, kIdS, 0u);
        mma_t_k64<D>(tmem + C::T_DP, tmem + C::T_DOHI, vl, kIdS, 1u);
        mma_t_k64<D>(tmem + C::T_DP, tmem + C::T_DOLO, vh, kIdS, 1u);
        mma_commit(bar(Q_DP_FULL));
      };
      for (uint32_t cons = 0; ok;) {
        const uint32_t sl = cons % kItemSlots;
        if (!mbar_wait(bar(Q_ITEM_FULL + sl), (cons / kItemSlots) & 1, ab, 133)) { ok = false; break; }
        const int idx = item_slot[sl];
        mbar_arrive(bar(Q_ITEM_EMPTY + sl));
        ++cons;
        if (idx >= n_items) break;
        const DqItem it = dq_decode(p, idx);
        int kb = dq_first(p, it);
        if (kb < 0) continue;
        // Q~ and dO rows in TMEM (written after the previous item's dQ~ was read)
        if (!mbar_wait(bar(Q_A_READY), arc & 1, ab, 134)) { ok = false; break; }
        ++arc;
        if (!wait_k(k_it)) { ok = false; break; }
        tc_fence_after();
        issue_s(k_it);
        issue_dp(k_it);
        bool first = true;
        while (kb >= 0) {
          const int kn = dq_next(p, it, kb);
          // S(next) once S(this) is in registers
          if (!mbar_wait(bar(Q_S_READ), s_read & 1, ab, 135)) { ok = false; break; }
          ++s_read;
          if (kn >= 0) {
            if (!wait_k(k_it + 1)) { ok = false; break; }
            tc_fence_after();
            issue_s(k_it + 1);
          }
          // dQ~ += dS K~ (dS hi/lo over dP), then dP(next) over it
          if (!mbar_wait(bar(Q_DS_FULL), ds_full & 1, ab, 136)) { ok = false; break; }
          ++ds_full;
          tc_fence_after();
          const uint64_t kh = mnmajor_desc_lbo(stage(k_it), kBox64),
                         kl = mnmajor_desc_lbo(stage(k_it) + C::kPlane, kBox64);
          mma_t_m64(tmem + C::T_DQ, tmem + C::T_DP, kh, kIdQ, first ? 0u : 1u);
          mma_t_m64(tmem + C::T_DQ, tmem + C::T_DP, kl, kIdQ, 1u);
          mma_t_m64(tmem + C::T_DQ, tmem + C::T_DP + 32u, kh, kIdQ, 1u);
          mma_commit(bar(Q_K_EMPTY + k_it % kSt));
          ++k_it;
          if (kn >= 0) issue_dp(k_it);
          first = false;
          kb = kn;
        }
        if (!ok) break;
        mma_commit(bar(Q_DQ_FULL));
      }
    }
  } else {
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;            // 32-key half of a 64-key block
    const int r = quarter * 32 + lane;           // TMEM lane = query row
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const size_t hstride = (size_t)p.n_tiles * 128;
    uint32_t s_full = 0, dp_full = 0, dq_full = 0;
    bool ok = true;
    for (uint32_t cons = 0; ok;) {
      const uint32_t sl = cons % kItemSlots;
      if (!__all_sync(0xffffffffu, mbar_wait(bar(Q_ITEM_FULL + sl), (cons / kItemSlots) & 1, ab, 137))) {
        ok = false;
        break;
      }
      const int idx = item_slot[sl];
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(Q_ITEM_EMPTY + sl));
      ++cons;
      if (idx >= n_items) break;
      const DqItem it = dq_decode(p, idx);
      const int64_t q = (int64_t)it.i * 128 + r;
      const bool q_ok = q < p.S;
      const int32_t seg_q = q_ok ? (p.seg ? p.seg[(size_t)it.b * p.S + q] : 0) : -1;
      const size_t tok = (size_t)it.b * p.S + (size_t)(q_ok ? q : 0);
      const size_t lrow = ((size_t)it.b * p.H + it.h) * hstride + (size_t)q;
      const float L2 = p.lse2[lrow];
      const float Dq = p.dpad[lrow];
      float* dqrow = p.out0 + (tok * p.H + it.h) * D + half * (D / 2);
      const int kb0 = dq_first(p, it);
      if (kb0 < 0) {
        if (q_ok) {
#pragma unroll
          for (int c = 0; c < D / 8; ++c)
            reinterpret_cast<float4*>(dqrow)[c] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        continue;
      }
      // this thread's half of the rows of Q~ hi/lo and dO hi/lo into TMEM
      {
        const size_t off = (tok * p.H + it.h) * D + half * (D / 2);
        const __nv_bfloat16* src[4] = {p.a_hi + off, p.a_lo + off, p.b_hi + off, p.b_lo + off};
        const uint32_t col[4] = {C::T_QHI, C::T_QLO, C::T_DOHI, C::T_DOLO};
#pragma unroll
        for (int pl = 0; pl < 4; ++pl) {
          const uint4* s4 = reinterpret_cast<const uint4*>(src[pl]);
          if constexpr (D == 128) {
            uint32_t v[32];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const uint4 a = q_ok ? s4[u] : make_uint4(0, 0, 0, 0);
              v[4 * u] = a.x; v[4 * u + 1] = a.y; v[4 * u + 2] = a.z; v[4 * u + 3] = a.w;
            }
            tmem_st32(tmem + lane_base + col[pl] + 32u * half, v);
          } else {
            uint32_t v[16];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const uint4 a = q_ok ? s4[u] : make_uint4(0, 0, 0, 0);
              v[4 * u] = a.x; v[4 * u + 1] = a.y; v[4 * u + 2] = a.z; v[4 * u + 3] = a.w;
            }
            tmem_st16(tmem + lane_base + col[pl] + 16u * half, v);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(Q_A_READY));
      }
      for (int kb = kb0; kb >= 0; kb = dq_next(p, it, kb)) {
        const int64_t k0 = (int64_t)kb * 64 + 32 * half;  // first key of this half
        bool partial = (p.causal && (int64_t)kb * 64 + 63 > (int64_t)it.i * 128) ||
                       ((int64_t)(kb + 1) * 64 > p.S) || ((int64_t)(it.i + 1) * 128 > p.S);
        if (p.seg) {
          const size_t kt = (size_t)it.b * p.n_tiles + (kb >> 1);
          const int32_t a0 = p.ktmin[kt], a1 = p.ktmax[kt];
          partial |= !(it.qmin >= 0 && it.qmin == it.qmax && a0 == it.qmin && a1 == it.qmin);
        }
        uint32_t mw = 0xffffffffu;
        if (partial) {
          int hi = 32;
          if (p.causal) {
            const int64_t d = q - k0 + 1;
            hi = d < 0 ? 0 : (d > 32 ? 32 : (int)d);
          }
          const int64_t kv = p.S - k0;
          const int kvalid = kv > 32 ? 32 : (kv < 0 ? 0 : (int)kv);
          if (kvalid < hi) hi = kvalid;
          if (seg_q < 0) hi = 0;
          uint32_t bits = bit_range(0, hi);
          if (p.seg) {
            const int32_t kid = lane < kvalid ? __ldg(p.kseg + (size_t)it.b * p.S + k0 + lane) : INT_MIN;
            bits &= warp_segment_bits(kid, seg_q);
          }
          mw = bits;
        }
        if (!__all_sync(0xffffffffu, mbar_wait(bar(Q_S_FULL), s_full & 1, ab, 138))) { ok = false; break; }
        ++s_full;
        tc_fence_after();
        float pr[32];
        {
          uint32_t sr[32];
          tmem_ld32(tmem + lane_base + C::T_S + 32u * half, sr);
          tmem_wait_ld();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(Q_S_READ));
#pragma unroll
          for (int c = 0; c < 32; ++c)
            pr[c] = ((mw >> c) & 1u) ? fast_exp2(fmaf(__uint_as_float(sr[c]), p.scale_log2, -L2)) : 0.f;
        }
        if (!__all_sync(0xffffffffu, mbar_wait(bar(Q_DP_FULL), dp_full & 1, ab, 139))) { ok = false; break; }
        ++dp_full;
        tc_fence_after();
        {
          uint32_t dr[32], dh[16], dl[16];
          const uint32_t tdp = tmem + lane_base + C::T_DP;
          tmem_ld32(tdp + 32u * half, dr);
          tmem_wait_ld();
#pragma unroll
          for (int u = 0; u < 16; ++u)
            split_pair(pr[2 * u] * (__uint_as_float(dr[2 * u]) - Dq),
                       pr[2 * u + 1] * (__uint_as_float(dr[2 * u + 1]) - Dq), &dh[u], &dl[u]);
          // every warp of this lane quarter has read dP before any writes over it
          named_bar_sync(1 + quarter, 64);
          tmem_st16(tdp + 16u * half, dh);
          tmem_st16(tdp + 32u + 16u * half, dl);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(Q_DS_FULL));
      }
      if (!ok) break;
      if (!__all_sync(0xffffffffu, mbar_wait(bar(Q_DQ_FULL), dq_full & 1, ab, 140))) { ok = false; break; }
      ++dq_full;
      tc_fence_after();
      // dq = R(p)^T scale dQ~ for this thread's D/2 columns
#pragma unroll 1
      for (int c = 0; c < D / 64; ++c) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_base + C::T_DQ + half * (D / 2) + 32u * c, v);
        tmem_wait_ld();
        float x[32];
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          float a = __uint_as_float(v[2 * u]) * p.scale, b = __uint_as_float(v[2 * u + 1]) * p.scale;
          if (p.rotate) {
            float cs, sn;
            rope_cos_sin_w(q, freq[half * (D / 4) + 16 * c + u], &cs, &sn);
            const float a2 = a * cs + b * sn, b2 = b * cs - a * sn;
            a = a2;
            b = b2;
          }
          x[2 * u] = a;
          x[2 * u + 1] = b;
        }
        if (q_ok) {
#pragma unroll
          for (int u = 0; u < 8; ++u)
            reinterpret_cast<float4*>(dqrow + 32 * c)[u] =
                make_float4(x[4 * u], x[4 * u + 1], x[4 * u + 2], x[4 * u + 3]);
        }
      }
      tc_fence_before();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    if (warp == 1 && lane == 0) {
      mma_commit(bar(Q_FIN));
      drain_wait(bar(Q_FIN), 0);
    }
    if (warp == 0 && lane == 0) {
      for (uint32_t n = (k_issued > (uint32_t)kSt ? k_issued - kSt : 0); n < k_issued; ++n)
        drain_wait(bar(Q_K_FULL + n % kSt), (n / kSt) & 1);
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ============================================================ dK/dV kernel
template <int D> struct KvCfg {
  static constexpr uint32_t kKPlane = kBox128 * (D / 64);  // 128 keys x D
  static constexpr uint32_t kPlane = kBox64 * (D / 64);    // 64 queries x D
  static constexpr uint32_t OFF_K = 0;                      // K~ hi, lo
  static constexpr uint32_t OFF_QD = 2 * kKPlane;           // 2 stages x (Q~ hi, lo, dO hi, lo)
  static constexpr uint32_t kStage = 4 * kPlane;
  static constexpr uint32_t OFF_SMALL = OFF_QD + 2 * kStage;
  static constexpr uint32_t SOFF_LD = 320;                  // 2 stages x (LSE2[64], D[64])
  static constexpr uint32_t kSmemBytes = OFF_SMALL + SOFF_LD + 2 * 512 + (D / 2) * 8 + 1024;
  static constexpr uint32_t T_VHI = 0, T_VLO = D / 2, T_S = D, T_DP = D + 64, T_DV = D + 128,
                            T_DK = 2 * D + 128;
};

enum : uint32_t {
  K_KV_FULL = 0, K_KV_EMPTY = 1,
  K_QD_FULL = 2, K_QD_EMPTY = 4,   // 2 stages
  K_A_READY = 6, K_S_FULL = 7, K_DP_FULL = 8, K_P_FULL = 9, K_DS_FULL = 10, K_DKV_FULL = 11,
  K_FIN = 12, K_ITEM_FULL = 13, K_ITEM_EMPTY = 17, K_COUNT = 21
};

struct KvItem {
  int b, h, j;
  int lo, hi;   // 64-query blocks
  int32_t kmin, kmax;
};

__device__ __forceinline__ KvItem kv_decode(const X3BwdParams& p, int idx) {
  KvItem it;
  const int bh = idx / p.n_tiles;
  it.j = idx % p.n_tiles;
  it.b = bh / p.H;
  it.h = bh % p.H;
  it.lo = p.causal ? 2 * it.j : 0;
  it.hi = p.n_b64 - 1;
  it.kmin = 0;
  it.kmax = 0;
  if (p.seg) {
    const size_t kj = (size_t)it.b * p.n_tiles + it.j;
    it.hi = min(2 * p.k_hi[kj] + 1, p.n_b64 - 1);
    it.kmin = p.ktmin[kj];
    it.kmax = p.ktmax[kj];
  }
  return it;
}

__device__ __forceinline__ bool kv_rel(const X3BwdParams& p, const KvItem& it, int qb) {
  if (qb < it.lo || qb > it.hi) return false;
  if (!p.seg) return true;
  const size_t qi = (size_t)it.b * p.n_tiles + (qb >> 1);
  return meet(it.kmin, it.kmax, p.tmin[qi], p.tmax[qi]);
}

__device__ __forceinline__ int kv_next(const X3BwdParams& p, const KvItem& it, int qb) {
  for (++qb; qb <= it.hi; ++qb)
    if (kv_rel(p, it, qb)) return qb;
  return -1;
}

__device__ __forceinline__ int kv_first(const X3BwdParams& p, const KvItem& it) {
  if (it.lo > it.hi) return -1;
  return kv_rel(p, it, it.lo) ? it.lo : kv_next(p, it, it.lo);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
attn_bwd_dkdv_x3_kernel(const __grid_constant__ CUtensorMap tm_khi, const __grid_constant__ CUtensorMap tm_klo,
                        const __grid_constant__ CUtensorMap tm_qhi, const __grid_constant__ CUtensorMap tm_qlo,
                        const __grid_constant__ CUtensorMap tm_dohi, const __grid_constant__ CUtensorMap tm_dolo,
                        const X3BwdParams p) {
  using C = KvCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  const uint32_t small = base + C::OFF_SMALL;
  auto bar = [&](uint32_t slot) { return small + 8u * slot; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_SMALL + 256 + 8);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_SMALL + 256);
  volatile int* item_slot = reinterpret_cast<volatile int*>(smem + C::OFF_SMALL + 256 + 16);
  const float* ld_smem = reinterpret_cast<const float*>(smem + C::OFF_SMALL + C::SOFF_LD);
  double* freq = reinterpret_cast<double*>(smem + C::OFF_SMALL + C::SOFF_LD + 2 * 512);
  int* item_counter = &p.status->item_counter[0];
  const Abort ab{abort_flag, p.status};
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_items = p.B * p.H * p.n_tiles;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(bar(K_KV_FULL), 1);
    mbar_init(bar(K_KV_EMPTY), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(K_QD_FULL + s), 1);
      mbar_init(bar(K_QD_EMPTY + s), 1);
    }
    mbar_init(bar(K_A_READY), kEWWarps);
    mbar_init(bar(K_S_FULL), 1);
    mbar_init(bar(K_DP_FULL), 1);
    mbar_init(bar(K_P_FULL), kEWWarps);
    mbar_init(bar(K_DS_FULL), kEWWarps);
    mbar_init(bar(K_DKV_FULL), 1);
    mbar_init(bar(K_FIN), 1);
    for (uint32_t sl = 0; sl < kItemSlots; ++sl) {
      mbar_init(bar(K_ITEM_FULL + sl), 1);
      mbar_init(bar(K_ITEM_EMPTY + sl), 1 + kEWWarps);
    }
    fence_mbar_init();
    tma_prefetch_desc(&tm_khi);
    tma_prefetch_desc(&tm_klo);
    tma_prefetch_desc(&tm_qhi);
    tma_prefetch_desc(&tm_qlo);
    tma_prefetch_desc(&tm_dohi);
    tma_prefetch_desc(&tm_dolo);
  }
  if (threadIdx.x >= 64 && threadIdx.x < 64 + D / 2 && p.rotate)
    freq[threadIdx.x - 64] = rope_freq(threadIdx.x - 64, D, p.log2_theta);
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  uint32_t kv_issued = 0, qd_issued = 0;

  if (warp == 0) {
    if (lane == 0) {
      uint32_t qd_it = 0;
      bool ok = true;
      const size_t hstride = (size_t)p.n_tiles * 128;
      for (uint32_t pub = 0; ok;) {
        const uint32_t sl = pub % kItemSlots;
        if (pub >= kItemSlots &&
            !mbar_wait(bar(K_ITEM_EMPTY + sl), ((pub / kItemSlots) - 1) & 1, ab, 150)) {
          ok = false;
          break;
        }
        const int idx = atomicAdd(item_counter, 1);
        item_slot[sl] = idx;
        mbar_arrive(bar(K_ITEM_FULL + sl));
        ++pub;
        if (idx >= n_items) break;
        const KvItem it = kv_decode(p, idx);
        int qb = kv_first(p, it);
        if (qb < 0) continue;
        if (kv_issued > 0 && !mbar_wait(bar(K_KV_EMPTY), (kv_issued - 1) & 1, ab, 151)) { ok = false; break; }
        mbar_expect_tx(bar(K_KV_FULL), 2 * C::kKPlane);
#pragma unroll
        for (int bx = 0; bx < D / 64; ++bx) {
          tma_load_4d(base + C::OFF_K + bx * kBox128, &tm_khi, bar(K_KV_FULL), 64 * bx, it.h, it.j * 128, it.b);
          tma_load_4d(base + C::OFF_K + C::kKPlane + bx * kBox128, &tm_klo, bar(K_KV_FULL), 64 * bx, it.h,
                      it.j * 128, it.b);
        }
        ++kv_issued;
        const float* lse2 = p.lse2 + ((size_t)it.b * p.H + it.h) * hstride;
        const float* dpad = p.dpad + ((size_t)it.b * p.H + it.h) * hstride;
        for (; qb >= 0 && ok; qb = kv_next(p, it, qb)) {
          const uint32_t s = qd_it & 1;
          if (!mbar_wait(bar(K_QD_EMPTY + s), ((qd_it >> 1) & 1) ^ 1, ab, 152)) { ok = false; break; }
          const uint32_t full = bar(K_QD_FULL + s);
          mbar_expect_tx(full, C::kStage + 512);
          const uint32_t dst = base + C::OFF_QD + s * C::kStage;
#pragma unroll
          for (int bx = 0; bx < D / 64; ++bx) {
            tma_load_4d(dst + bx * kBox64, &tm_qhi, full, 64 * bx, it.h, qb * 64, it.b);
            tma_load_4d(dst + C::kPlane + bx * kBox64, &tm_qlo, full, 64 * bx, it.h, qb * 64, it.b);
            tma_load_4d(dst + 2 * C::kPlane + bx * kBox64, &tm_dohi, full, 64 * bx, it.h, qb * 64, it.b);
            tma_load_4d(dst + 3 * C::kPlane + bx * kBox64, &tm_dolo, full, 64 * bx, it.h, qb * 64, it.b);
          }
          const uint32_t ld = small + C::SOFF_LD + s * 512;
          bulk_load(ld, lse2 + (size_t)qb * 64, 256, full);
          bulk_load(ld + 256, dpad + (size_t)qb * 64, 256, full);
          qd_issued = ++qd_it;
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t kIdS = idesc_bf16(128, 64, 0, 0);   // K-major x K-major, N = 64
      constexpr uint32_t kIdG = idesc_bf16(128, D, 0, 1);    // TMEM x MN-major, N = D
      uint32_t qd_it = 0, kv_items = 0, arc = 0, pf = 0, dsf = 0, dkv = 0;
      bool ok = true;
      const uint64_t kh = kmajor_desc(base + C::OFF_K), kl = kmajor_desc(base + C::OFF_K + C::kKPlane);
      auto stage = [&](uint32_t n) { return base + C::OFF_QD + (n & 1) * C::kStage; };
      auto wait_qd = [&](uint32_t n) {
        return mbar_wait(bar(K_QD_FULL + (n & 1)), (n >> 1) & 1, ab, 153);
      };
      auto issue_s = [&](uint32_t n) {
        const uint64_t qh = kmajor_desc(stage(n)), ql = kmajor_desc(stage(n) + C::kPlane);
        mma_s128_k64<D>(tmem + C::T_S, kh, qh, kIdS, 0u);
        mma_s128_k64<D>(tmem + C::T_S, kh, ql, kIdS, 1u);
        mma_s128_k64<D>(tmem + C::T_S, kl, qh, kIdS, 1u);
        mma_commit(bar(K_S_FULL));
      };
      auto issue_dp = [&](uint32_t n) {
        const uint64_t dh = kmajor_desc(stage(n) + 2 * C::kPlane),
                       dl = kmajor_desc(stage(n) + 3 * C::kPlane);
        mma_t_k64<D>(tmem + C::T_DP, tmem + C::T_VHI, dh, kIdS, 0u);
        mma_t_k64<D>(tmem + C::T_DP, tmem + C::T_VHI, dl, kIdS, 1u);
        mma_t_k64<D>(tmem + C::T_DP, tmem + C::T_VLO, dh, kIdS, 1u);
        mma_commit(bar(K_DP_FULL));
      };
      for (uint32_t cons = 0; ok;) {
        const uint32_t sl = cons % kItemSlots;
        if (!mbar_wait(bar(K_ITEM_FULL + sl), (cons / kItemSlots) & 1, ab, 154)) { ok = false; break; }
        const int idx = item_slot[sl];
        mbar_arrive(bar(K_ITEM_EMPTY + sl));
        ++cons;
        if (idx >= n_items) break;
        const KvItem it = kv_decode(p, idx);
        int qb = kv_first(p, it);
        if (qb < 0) continue;
        if (!mbar_wait(bar(K_KV_FULL), kv_items & 1, ab, 155)) { ok = false; break; }
        ++kv_items;
        // V hi/lo rows in TMEM (written after the previous item's dK, dV were read)
        if (!mbar_wait(bar(K_A_READY), arc & 1, ab, 156)) { ok = false; break; }
        ++arc;
        if (!wait_qd(qd_it)) { ok = false; break; }
        tc_fence_after();
        issue_s(qd_it);
        issue_dp(qd_it);
        bool first = true;
        while (qb >= 0) {
          const int qn = kv_next(p, it, qb);
          // dV += P^T dO (P^T hi/lo over S^T), then S^T(next) over it
          if (!mbar_wait(bar(K_P_FULL), pf & 1, ab, 157)) { ok = false; break; }
          ++pf;
          tc_fence_after();
          const uint64_t oh = mnmajor_desc_lbo(stage(qd_it) + 2 * C::kPlane, kBox64),
                         ol = mnmajor_desc_lbo(stage(qd_it) + 3 * C::kPlane, kBox64);
          mma_t_m64(tmem + C::T_DV, tmem + C::T_S, oh, kIdG, first ? 0u : 1u);
          mma_t_m64(tmem + C::T_DV, tmem + C::T_S, ol, kIdG, 1u);
          mma_t_m64(tmem + C::T_DV, tmem + C::T_S + 32u, oh, kIdG, 1u);
          if (qn >= 0) {
            if (!wait_qd(qd_it + 1)) { ok = false; break; }
            tc_fence_after();
            issue_s(qd_it + 1);
          }
          // dK~ += dS^T Q~ (dS^T hi/lo over dP^T), then dP^T(next) over it
          if (!mbar_wait(bar(K_DS_FULL), dsf & 1, ab, 158)) { ok = false; break; }
          ++dsf;
          tc_fence_after();
          const uint64_t qh = mnmajor_desc_lbo(stage(qd_it), kBox64),
                         ql = mnmajor_desc_lbo(stage(qd_it) + C::kPlane, kBox64);
          mma_t_m64(tmem + C::T_DK, tmem + C::T_DP, qh, kIdG, first ? 0u : 1u);
          mma_t_m64(tmem + C::T_DK, tmem + C::T_DP, ql, kIdG, 1u);
          mma_t_m64(tmem + C::T_DK, tmem + C::T_DP + 32u, qh, kIdG, 1u);
          mma_commit(bar(K_QD_EMPTY + (qd_it & 1)));
          ++qd_it;
          if (qn >= 0) issue_dp(qd_it);
          first = false;
          qb = qn;
        }
        if (!ok) break;
        mma_commit(bar(K_DKV_FULL));
        mma_commit(bar(K_KV_EMPTY));
        ++dkv;
      }
    }
  } else {
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;            // 32-query half of a 64-query block
    const int r = quarter * 32 + lane;           // TMEM lane = key row
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    uint32_t steps = 0, s_full = 0, dp_full = 0, dkv = 0;
    bool ok = true;
    for (uint32_t cons = 0; ok;) {
      const uint32_t sl = cons % kItemSlots;
      if (!__all_sync(0xffffffffu, mbar_wait(bar(K_ITEM_FULL + sl), (cons / kItemSlots) & 1, ab, 159))) {
        ok = false;
        break;
      }
      const int idx = item_slot[sl];
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(K_ITEM_EMPTY + sl));
      ++cons;
      if (idx >= n_items) break;
      const KvItem it = kv_decode(p, idx);
      const int64_t key = (int64_t)it.j * 128 + r;
      const bool key_ok = key < p.S;
      const int32_t seg_k = key_ok ? (p.seg ? p.kseg[(size_t)it.b * p.S + key] : 0) : -1;
      const size_t tok = (size_t)it.b * p.S + (size_t)(key_ok ? key : 0);
      float* dkrow = p.out0 + (tok * p.H + it.h) * D + half * (D / 2);
      float* dvrow = p.out1 + (tok * p.H + it.h) * D + half * (D / 2);
      const int qb0 = kv_first(p, it);
      if (qb0 < 0) {
        if (key_ok) {
#pragma unroll
          for (int c = 0; c < D / 8; ++c) {
            reinterpret_cast<float4*>(dkrow)[c] = make_float4(0.f, 0.f, 0.f, 0.f);
            reinterpret_cast<float4*>(dvrow)[c] = make_float4(0.f, 0.f, 0.f, 0.f);
          }
        }
        continue;
      }
      // this thread's half of the row of V hi/lo into TMEM
      {
        const size_t off = (tok * p.H + it.h) * D + half * (D / 2);
        const __nv_bfloat16* src[2] = {p.a_hi + off, p.a_lo + off};
        const uint32_t col[2] = {C::T_VHI, C::T_VLO};
#pragma unroll
        for (int pl = 0; pl < 2; ++pl) {
          const uint4* s4 = reinterpret_cast<const uint4*>(src[pl]);
          if constexpr (D == 128) {
            uint32_t v[32];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const uint4 a = key_ok ? s4[u] : make_uint4(0, 0, 0, 0);
              v[4 * u] = a.x; v[4 * u + 1] = a.y; v[4 * u + 2] = a.z; v[4 * u + 3] = a.w;
            }
            tmem_st32(tmem + lane_base + col[pl] + 32u * half, v);
          } else {
            uint32_t v[16];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const uint4 a = key_ok ? s4[u] : make_uint4(0, 0, 0, 0);
              v[4 * u] = a.x; v[4 * u + 1] = a.y; v[4 * u + 2] = a.z; v[4 * u + 3] = a.w;
            }
            tmem_st16(tmem + lane_base + col[pl] + 16u * half, v);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(K_A_READY));
      }
      for (int qb = qb0; qb >= 0; qb = kv_next(p, it, qb)) {
        const int64_t q0 = (int64_t)qb * 64 + 32 * half;   // first query of this half
        bool partial = (p.causal && (int64_t)it.j * 128 + 127 > (int64_t)qb * 64) ||
                       ((int64_t)(qb + 1) * 64 > p.S) || ((int64_t)(it.j + 1) * 128 > p.S);
        if (p.seg) {
          const size_t qi = (size_t)it.b * p.n_tiles + (qb >> 1);
          const int32_t a0 = p.tmin[qi], a1 = p.tmax[qi];
          partial |= !(it.kmin >= 0 && it.kmin == it.kmax && a0 == it.kmin && a1 == it.kmin);
        }
        uint32_t mw = 0xffffffffu;
        if (partial) {
          int lo = 0;
          if (p.causal) {
            const int64_t d = key - q0;
            lo = d < 0 ? 0 : (d > 32 ? 32 : (int)d);
          }
          const int64_t qv = p.S - q0;
          const int hi = qv > 32 ? 32 : (qv < 0 ? 0 : (int)qv);
          uint32_t bits = seg_k >= 0 ? bit_range(lo, hi) : 0u;
          if (p.seg) {
            const int32_t qseg = lane < hi ? __ldg(p.seg + (size_t)it.b * p.S + q0 + lane) : INT_MIN;
            bits &= warp_segment_bits(qseg, seg_k);
          }
          mw = bits;
        }
        const uint32_t stg = steps & 1;
        const float* lse2 = ld_smem + stg * 128 + 32 * half;
        const float* dsum = lse2 + 64;
        if (!__all_sync(0xffffffffu, mbar_wait(bar(K_S_FULL), s_full & 1, ab, 160) &&
                                         mbar_wait(bar(K_QD_FULL + stg), (steps >> 1) & 1, ab, 161))) {
          ok = false;
          break;
        }
        ++s_full;
        tc_fence_after();
        float pr[32];
        {
          uint32_t sr[32], ph[16], pl[16];
          const uint32_t ts = tmem + lane_base + C::T_S;
          tmem_ld32(ts + 32u * half, sr);
          tmem_wait_ld();
          const float4* l4 = reinterpret_cast<const float4*>(lse2);
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const float4 L = l4[u];
            const float Ls[4] = {L.x, L.y, L.z, L.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int c = 4 * u + e;
              pr[c] = ((mw >> c) & 1u) ? fast_exp2(fmaf(__uint_as_float(sr[c]), p.scale_log2, -Ls[e])) : 0.f;
            }
          }
#pragma unroll
          for (int u = 0; u < 16; ++u) split_pair(pr[2 * u], pr[2 * u + 1], &ph[u], &pl[u]);
          // every warp of this lane quarter has read S^T before any writes over it
          named_bar_sync(1 + quarter, 64);
          tmem_st16(ts + 16u * half, ph);
          tmem_st16(ts + 32u + 16u * half, pl);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(K_P_FULL));
        if (!__all_sync(0xffffffffu, mbar_wait(bar(K_DP_FULL), dp_full & 1, ab, 162))) { ok = false; break; }
        ++dp_full;
        tc_fence_after();
        {
          uint32_t dr[32], dh[16], dl[16];
          const uint32_t tdp = tmem + lane_base + C::T_DP;
          tmem_ld32(tdp + 32u * half, dr);
          tmem_wait_ld();
          const float4* d4 = reinterpret_cast<const float4*>(dsum);
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const float4 Dv = d4[u];
            const float* pp = pr + 4 * u;
            split_pair(pp[0] * (__uint_as_float(dr[4 * u]) - Dv.x),
                       pp[1] * (__uint_as_float(dr[4 * u + 1]) - Dv.y), &dh[2 * u], &dl[2 * u]);
            split_pair(pp[2] * (__uint_as_float(dr[4 * u + 2]) - Dv.z),
                       pp[3] * (__uint_as_float(dr[4 * u + 3]) - Dv.w), &dh[2 * u + 1], &dl[2 * u + 1]);
          }
          named_bar_sync(1 + quarter, 64);
          tmem_st16(tdp + 16u * half, dh);
          tmem_st16(tdp + 32u + 16u * half, dl);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(K_DS_FULL));
        ++steps;
      }
      if (!ok) break;
      if (!__all_sync(0xffffffffu, mbar_wait(bar(K_DKV_FULL), dkv & 1, ab, 163))) { ok = false; break; }
      ++dkv;
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < D / 64; ++c) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_base + C::T_DV + half * (D / 2) + 32u * c, v);
        tmem_wait_ld();
        if (key_ok) {
#pragma unroll
          for (int u = 0; u < 8; ++u)
            reinterpret_cast<float4*>(dvrow + 32 * c)[u] =
                make_float4(__uint_as_float(v[4 * u]), __uint_as_float(v[4 * u + 1]),
                            __uint_as_float(v[4 * u + 2]), __uint_as_float(v[4 * u + 3]));
        }
        tmem_ld32(tmem + lane_base + C::T_DK + half * (D / 2) + 32u * c, v);
        tmem_wait_ld();
        float x[32];
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          float a = __uint_as_float(v[2 * u]) * p.scale, b = __uint_as_float(v[2 * u + 1]) * p.scale;
          if (p.rotate) {
            float cs, sn;
            rope_cos_sin_w(key, freq[half * (D / 4) + 16 * c + u], &cs, &sn);
            const float a2 = a * cs + b * sn, b2 = b * cs - a * sn;
            a = a2;
            b = b2;
          }
          x[2 * u] = a;
          x[2 * u + 1] = b;
        }
        if (key_ok) {
#pragma unroll
          for (int u = 0; u < 8; ++u)
            reinterpret_cast<float4*>(dkrow + 32 * c)[u] =
                make_float4(x[4 * u], x[4 * u + 1], x[4 * u + 2], x[4 * u + 3]);
        }
      }
      tc_fence_before();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    if (warp == 1 && lane == 0) {
      mma_commit(bar(K_FIN));
      drain_wait(bar(K_FIN), 0);
    }
    if (warp == 0 && lane == 0) {
      if (kv_issued > 0) drain_wait(bar(K_KV_FULL), (kv_issued - 1) & 1);
      for (uint32_t n = (qd_issued > 2 ? qd_issued - 2 : 0); n < qd_issued; ++n)
        drain_wait(bar(K_QD_FULL + (n & 1)), (n >> 1) & 1);
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

X3BwdParams make_params(const Problem& pb, const Workspace& ws) {
  X3BwdParams p{};
  p.seg = pb.seg;
  p.kseg = pb.kseg;
  p.tmin = ws.tile_min;
  p.tmax = ws.tile_max;
  p.ktmin = ws.ktile_min;
  p.ktmax = ws.ktile_max;
  p.q_lo = ws.q_lo;
  p.k_hi = ws.k_hi;
  p.lse2 = ws.lse2_pad;
  p.dpad = ws.delta_pad;
  p.status = ws.status;
  p.S = pb.S;
  p.H = (int)pb.H;
  p.B = (int)pb.B;
  p.n_tiles = (int)pb.n_tiles;
  p.n_b64 = (int)((pb.S + 63) / 64);
  p.scale = pb.scale;
  p.scale_log2 = pb.scale * 1.4426950408889634f;
  p.causal = pb.causal;
  p.rotate = pb.theta > 0.0;
  p.log2_theta = p.rotate ? log2(pb.theta) : 0.0;
  return p;
}

template <int D>
cudaError_t launch_dkdv(const Problem& pb, const Workspace& ws, float* dk, float* dv, cudaStream_t st) {
  CUtensorMap khi, klo, qhi, qlo, dohi, dolo;
  if (!make_bf16_map(&khi, ws.kx_hi, pb.B, pb.S, pb.H, D, 128) ||
      !make_bf16_map(&klo, ws.kx_lo, pb.B, pb.S, pb.H, D, 128) ||
      !make_bf16_map(&qhi, ws.qx_hi, pb.B, pb.S, pb.H, D, 64) ||
      !make_bf16_map(&qlo, ws.qx_lo, pb.B, pb.S, pb.H, D, 64) ||
      !make_bf16_map(&dohi, ws.dox_hi, pb.B, pb.S, pb.H, D, 64) ||
      !make_bf16_map(&dolo, ws.dox_lo, pb.B, pb.S, pb.H, D, 64))
    return cudaErrorInvalidValue;
  X3BwdParams p = make_params(pb, ws);
  p.a_hi = static_cast<const __nv_bfloat16*>(ws.vx_hi);
  p.a_lo = static_cast<const __nv_bfloat16*>(ws.vx_lo);
  p.out0 = dk;
  p.out1 = dv;
  using C = KvCfg<D>;
  static std::once_flag once;
  static cudaError_t err = cudaSuccess;
  std::call_once(once, [] {
    err = cudaFuncSetAttribute(attn_bwd_dkdv_x3_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)C::kSmemBytes);
  });
  if (err != cudaSuccess) return err;
  const int64_t n_items = pb.B * pb.H * pb.n_tiles;
  const int grid = (int)(n_items < sm_count() ? n_items : sm_count());
  attn_bwd_dkdv_x3_kernel<D><<<grid, kThreads, C::kSmemBytes, st>>>(khi, klo, qhi, qlo, dohi, dolo, p);
  note_launches(1);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_dq(const Problem& pb, const Workspace& ws, float* dq, cudaStream_t st) {
  CUtensorMap khi, klo, vhi, vlo;
  if (!make_bf16_map(&khi, ws.kx_hi, pb.B, pb.S, pb.H, D, 64) ||
      !make_bf16_map(&klo, ws.kx_lo, pb.B, pb.S, pb.H, D, 64) ||
      !make_bf16_map(&vhi, ws.vx_hi, pb.B, pb.S, pb.H, D, 64) ||
      !make_bf16_map(&vlo, ws.vx_lo, pb.B, pb.S, pb.H, D, 64))
    return cudaErrorInvalidValue;
  X3BwdParams p = make_params(pb, ws);
  p.a_hi = static_cast<const __nv_bfloat16*>(ws.qx_hi);
  p.a_lo = static_cast<const __nv_bfloat16*>(ws.qx_lo);
  p.b_hi = static_cast<const __nv_bfloat16*>(ws.dox_hi);
  p.b_lo = static_cast<const __nv_bfloat16*>(ws.dox_lo);
  p.out0 = dq;
  using C = DqCfg<D>;
  static std::once_flag once;
  static cudaError_t err = cudaSuccess;
  std::call_once(once, [] {
    err = cudaFuncSetAttribute(attn_bwd_dq_x3_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)C::kSmemBytes);
  });
  if (err != cudaSuccess) return err;
  const int64_t n_items = pb.B * pb.H * pb.n_tiles;
  const int grid = (int)(n_items < sm_count() ? n_items : sm_count());
  attn_bwd_dq_x3_kernel<D><<<grid, kThreads, C::kSmemBytes, st>>>(khi, klo, vhi, vlo, p);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_sm100_bwd_x3(const Problem& pb, const Workspace& ws, void* dq, void* dk, void* dv,
                                cudaStream_t st) {
  if (pb.B * pb.H * pb.n_tiles == 0) return cudaSuccess;
  float* fq = static_cast<float*>(dq);
  float* fk = static_cast<float*>(dk);
  float* fv = static_cast<float*>(dv);
  cudaError_t e;
  if (pb.D == 128) {
    e = launch_dkdv<128>(pb, ws, fk, fv, st);
    if (e == cudaSuccess) e = launch_dq<128>(pb, ws, fq, st);
  } else if (pb.D == 64) {
    e = launch_dkdv<64>(pb, ws, fk, fv, st);
    if (e == cudaSuccess) e = launch_dq<64>(pb, ws, fq, st);
  } else {
    e = cudaErrorInvalidValue;
  }
  return e;
}

}  // namespace lwm
