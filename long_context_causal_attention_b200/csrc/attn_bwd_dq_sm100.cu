// Backward attention, part 2 of 2: dQ, on the 5th-generation tensor cores
// (sm_100a), bf16, D=128.
//
// Per (query tile i, key tile j), recomputing P from the saved LSE (the
// FlashAttention recipe the paper card's references name):
//   S  = Q~_i K~_j^T        P  = exp(S * scale - LSE_i)
//   dP = dO_i V_j^T         dS = P o (dP - D_i),  D_i = dO_i . O_i
//   dQ~_i += dS K~_j        dq_i = R(p)^T scale dQ~_i
// One persistent CTA per SM owns a query tile i of one (b, h) and sweeps the
// key tiles j it may attend to; dQ~_i accumulates in tensor memory, and the
// epilogue applies the scale and the inverse rotation and writes bf16 dq, so
// no partial sums leave the CTA.  Q~_i and dO_i are the A operands of S and
// dP for the whole sweep, so they sit in tensor memory and every product of
// the sweep reads only its B operand (K~_j or V_j) from shared memory.
// Roles (576 threads; fewer control warps leave more registers to the
// element-wise ones):
//   warp 0      TMA producer: K~_j and V_j per step, 3-stage rings, K issued
//               two tiles ahead of V.
//   warp 1      MMA issuer (one thread); the whole warp allocates and frees
//               the tensor memory.
//   warps 2-17  element-wise work, four groups of four warps (one per TMEM
//               lane quarter, warp % 4) on 32 key columns each
//               (one query row per thread): Q~_i / dO_i rows into tensor
//               memory at the start of an item, P and dS per step, then the
//               dq epilogue.
// TMEM columns: S [0,128), dP [128,256) with dS (bf16) over it (each quarter
// packs its dS into the first 16 of its own 32 columns), dQ~ [256,384),
// Q~_i [384,448), dO_i [448,512) (bf16, two per column).
// MMA issue order per step:
//   S(j+1) once S(j) is in registers | dQ(j) after dS(j) | dP(j+1) ...
#include <cuda.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace lwm {

bool make_qkv_map(CUtensorMap* map, const void* ptr, int64_t B, int64_t S, int64_t H, int64_t D);
int sm_count();

namespace {

using namespace sm100;

constexpr int kD = 128;
constexpr int kThreads = 576;   // 2 control warps + 4 element-wise warpgroups
constexpr int kEW = 512;        // element-wise threads
constexpr uint32_t kTileBytes = 128 * kD * 2;
constexpr uint32_t kBoxBytes = kTileBytes / 2;

constexpr uint32_t SOFF_BAR = 0;
constexpr uint32_t SOFF_MISC = 256;
constexpr uint32_t SOFF_FREQ = 320;  // 64 RoPE frequencies, fp64
constexpr uint32_t kSmallBytes = SOFF_FREQ + (kD / 2) * 8;
constexpr int kKStages = 3;
constexpr int kVStages = 3;
constexpr uint32_t OFF_K = 0;
constexpr uint32_t OFF_V = OFF_K + kKStages * kTileBytes;
constexpr uint32_t kTilesBytes = OFF_V + kVStages * kTileBytes;  // 192 KB
constexpr uint32_t kSmemBytes = kTilesBytes + kSmallBytes + 1024;

enum : uint32_t {
  B_K_FULL = 0,    // kKStages
  B_K_EMPTY = 3,   // kKStages
  B_V_FULL = 6,    // kVStages
  B_V_EMPTY = 9,   // kVStages
  B_Q_READY = 12, B_S_FULL = 13, B_S_READ = 14, B_DP_FULL = 15, B_DS_FULL = 16,
  B_DQ_FULL = 17, B_DQ_EMPTY = 18, B_FIN = 19,
  B_ITEM_FULL = 20,   // 4 slots
  B_ITEM_EMPTY = 24   // 4 slots
};
constexpr uint32_t kItemSlots = 4;

struct DqParams {
  const int32_t* seg;    // query segment ids [B, S] or null
  const int32_t* kseg;   // key segment ids (seg unless a block pair)
  const int32_t* tmin;   // query tile bounds
  const int32_t* tmax;
  const int32_t* ktmin;  // key tile bounds
  const int32_t* ktmax;
  const int32_t* q_lo;
  const float* lse2;   // [B, H, nT*128]: LSE * log2(e), +inf where the row has no keys
  const float* dpad;   // [B, H, nT*128]: dot(dO, O), 0 past the end
  const __nv_bfloat16* q_rot;  // [B, S, H, D] rotated q
  const __nv_bfloat16* d_o;    // [B, S, H, D]
  __nv_bfloat16* dq;
  DeviceStatus* status;
  int64_t S;
  int H, B, n_tiles;
  float scale, scale_log2;
  int causal, rotate;
  double log2_theta;
};

struct Item {
  int b, h, i;
  int lo, hi;          // key tile range
  int32_t qmin, qmax;  // query tile id range
};

__device__ __forceinline__ bool meet(int32_t a0, int32_t a1, int32_t b0, int32_t b1) {
  return a1 >= 0 && b1 >= 0 && a0 <= b1 && b0 <= a1;
}

__device__ __forceinline__ Item decode(const DqParams& p, int idx) {
  Item it;
  const int bh = idx / p.n_tiles;
  it.i = p.n_tiles - 1 - (idx % p.n_tiles);  // most key tiles first (causal)
  it.b = bh / p.H;
  it.h = bh % p.H;
  it.lo = 0;
  it.hi = p.causal ? it.i : p.n_tiles - 1;
  it.qmin = 0;
  it.qmax = 0;
  if (p.seg) {
    const size_t qi = (size_t)it.b * p.n_tiles + it.i;
    it.lo = p.q_lo[qi];
    it.qmin = p.tmin[qi];
    it.qmax = p.tmax[qi];
  }
  return it;
}

__device__ __forceinline__ bool rel(const DqParams& p, const Item& it, int j) {
  if (j < it.lo || j > it.hi) return false;
  if (!p.seg) return true;
  const size_t kj = (size_t)it.b * p.n_tiles + j;
  return meet(it.qmin, it.qmax, p.ktmin[kj], p.ktmax[kj]);
}

__device__ __forceinline__ int next_rel(const DqParams& p, const Item& it, int j) {
  for (++j; j <= it.hi; ++j)
    if (rel(p, it, j)) return j;
  return -1;
}

__device__ __forceinline__ int first_rel(const DqParams& p, const Item& it) {
  if (it.lo > it.hi) return -1;
  return rel(p, it, it.lo) ? it.lo : next_rel(p, it, it.lo);
}

__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try(bar, parity)) {
    if (clock64() - t0 > kWaitCycles) return;
  }
}

__global__ void __launch_bounds__(kThreads, 1)
attn_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                   const DqParams p) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + kSmallBytes + 1023u) & ~1023u;
  const uint32_t bar0 = raw + SOFF_BAR;
  auto bar = [&](uint32_t slot) { return bar0 + 8u * slot; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem_raw + SOFF_MISC + 8);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem_raw + SOFF_MISC);
  double* freq = reinterpret_cast<double*>(smem_raw + SOFF_FREQ);
  // work items come from a global counter (greedy, in cost order): the TMA
  // thread takes one and publishes it to the CTA through a 4-slot ring
  volatile int* item_slot = reinterpret_cast<volatile int*>(smem_raw + SOFF_MISC + 16);
  int* item_counter = &p.status->item_counter[1];
  const Abort ab{abort_flag, p.status};
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_items = p.B * p.H * p.n_tiles;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(bar(B_K_FULL + s), 1);
      mbar_init(bar(B_K_EMPTY + s), 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(bar(B_V_FULL + s), 1);
      mbar_init(bar(B_V_EMPTY + s), 1);
    }
    mbar_init(bar(B_Q_READY), kEW / 32);
    mbar_init(bar(B_S_FULL), 1);
    mbar_init(bar(B_S_READ), kEW / 32);
    mbar_init(bar(B_DP_FULL), 1);
    mbar_init(bar(B_DS_FULL), kEW / 32);
    mbar_init(bar(B_DQ_FULL), 1);
    mbar_init(bar(B_DQ_EMPTY), kEW / 32);
    mbar_init(bar(B_FIN), 1);
    for (uint32_t sl = 0; sl < kItemSlots; ++sl) {
      mbar_init(bar(B_ITEM_FULL + sl), 1);
      mbar_init(bar(B_ITEM_EMPTY + sl), 1 + kEW / 32);
    }
    fence_mbar_init();
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (threadIdx.x >= 64 && threadIdx.x < 64 + kD / 2 && p.rotate)
    freq[threadIdx.x - 64] = rope_freq(threadIdx.x - 64, kD, p.log2_theta);
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
            !mbar_wait(bar(B_ITEM_EMPTY + sl), ((pub / kItemSlots) - 1) & 1, ab, 49)) {
          ok = false;
          break;
        }
        const int idx = atomicAdd(item_counter, 1);
        item_slot[sl] = idx;
        mbar_arrive(bar(B_ITEM_FULL + sl));
        ++pub;
        if (idx >= n_items) break;
        const Item it = decode(p, idx);
        auto load_k = [&](int j) -> bool {
          const uint32_t s = k_it % kKStages, n = k_it / kKStages;
          if (!mbar_wait(bar(B_K_EMPTY + s), (n & 1) ^ 1, ab, 52)) return false;
          mbar_expect_tx(bar(B_K_FULL + s), kTileBytes);
          const uint32_t dst = base + OFF_K + s * kTileBytes;
          tma_load_4d(dst, &tm_k, bar(B_K_FULL + s), 0, it.h, j * 128, it.b);
          tma_load_4d(dst + kBoxBytes, &tm_k, bar(B_K_FULL + s), 64, it.h, j * 128, it.b);
          k_issued = ++k_it;
          return true;
        };
        auto load_v = [&](int j) -> bool {
          const uint32_t s = v_it % kVStages, n = v_it / kVStages;
          if (!mbar_wait(bar(B_V_EMPTY + s), (n & 1) ^ 1, ab, 50)) return false;
          mbar_expect_tx(bar(B_V_FULL + s), kTileBytes);
          const uint32_t dst = base + OFF_V + s * kTileBytes;
          tma_load_4d(dst, &tm_v, bar(B_V_FULL + s), 0, it.h, j * 128, it.b);
          tma_load_4d(dst + kBoxBytes, &tm_v, bar(B_V_FULL + s), 64, it.h, j * 128, it.b);
          v_issued = ++v_it;
          return true;
        };
        // K runs two tiles ahead of V in issue order
        int jk = first_rel(p, it);
        for (int a = 0; a < 2 && jk >= 0 && ok; ++a, jk = next_rel(p, it, jk)) ok = load_k(jk);
        for (int j = first_rel(p, it); j >= 0 && ok; j = next_rel(p, it, j)) {
          ok = load_v(j);
          if (ok && jk >= 0) {
            ok = load_k(jk);
            jk = next_rel(p, it, jk);
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA
    if (lane == 0) {
      constexpr uint32_t kIdTK = idesc_bf16(128, 128, 0, 0);   // TMEM (K-major) x K-major
      constexpr uint32_t kIdTM = idesc_bf16(128, 128, 0, 1);   // TMEM (K-major) x MN-major
      const uint32_t tS = tmem, tDP = tmem + 128, tDQ = tmem + 256, tQ = tmem + 384,
                     tDO = tmem + 448;
      uint32_t k_it = 0, v_it = 0, steps = 0, dqc = 0, qrc = 0;
      bool ok = true;
      auto sk_of = [&](uint32_t n) { return base + OFF_K + (n % kKStages) * kTileBytes; };
      auto sv_of = [&](uint32_t n) { return base + OFF_V + (n % kVStages) * kTileBytes; };
      auto wait_k = [&](uint32_t n) {
        return mbar_wait(bar(B_K_FULL + n % kKStages), (n / kKStages) & 1, ab, 54);
      };
      auto issue_s = [&](uint32_t n) {
        mma_tk128(tS, tQ, kmajor_desc(sk_of(n)), kIdTK, 0u);
        mma_commit(bar(B_S_FULL));
      };
      // dP(j) with the next V tile; V_j is free again once dP(j) completes
      auto issue_dp = [&]() -> bool {
        if (!mbar_wait(bar(B_V_FULL + v_it % kVStages), (v_it / kVStages) & 1, ab, 56)) return false;
        tc_fence_after();
        mma_tk128(tDP, tDO, kmajor_desc(sv_of(v_it)), kIdTK, 0u);
        mma_commit(bar(B_DP_FULL));
        mma_commit(bar(B_V_EMPTY + v_it % kVStages));
        ++v_it;
        return true;
      };
      for (uint32_t cons = 0; ok;) {
        const uint32_t sl = cons % kItemSlots;
        if (!mbar_wait(bar(B_ITEM_FULL + sl), (cons / kItemSlots) & 1, ab, 48)) { ok = false; break; }
        const int idx = item_slot[sl];
        mbar_arrive(bar(B_ITEM_EMPTY + sl));
        ++cons;
        if (idx >= n_items) break;
        const Item it = decode(p, idx);
        int j = first_rel(p, it);
        if (j < 0) continue;  // nothing to do: the element-wise warps write zeros
        bool first = true;
        // Q~_i and dO_i in tensor memory (and the previous item's dQ read out)
        if (!mbar_wait(bar(B_Q_READY), qrc & 1, ab, 53)) { ok = false; break; }
        ++qrc;
        if (!wait_k(k_it)) { ok = false; break; }
        tc_fence_after();
        issue_s(k_it);
        if (!issue_dp()) { ok = false; break; }
        while (j >= 0) {
          const int jn = next_rel(p, it, j);
          // S(j+1) as soon as S(j) is in the element-wise warps' registers
          if (!mbar_wait(bar(B_S_READ), steps & 1, ab, 55)) { ok = false; break; }
          if (jn >= 0) {
            if (!wait_k(k_it + 1)) { ok = false; break; }
            tc_fence_after();
            issue_s(k_it + 1);
          }
          if (!mbar_wait(bar(B_DS_FULL), steps & 1, ab, 57)) { ok = false; break; }
          if (first && dqc > 0 && !mbar_wait(bar(B_DQ_EMPTY), (dqc - 1) & 1, ab, 58)) { ok = false; break; }
          tc_fence_after();
          mma_tm128<true>(tDQ, tDP, mnmajor_desc(sk_of(k_it)), kIdTM, first ? 0u : 1u);
          mma_commit(bar(B_K_EMPTY + k_it % kKStages));
          ++k_it;
          // dP(j+1): dS(j) in these columns went to dQ(j) just before (issue order)
          if (jn >= 0 && !issue_dp()) { ok = false; break; }
          ++steps;
          first = false;
          j = jn;
        }
        if (!ok) break;
        mma_commit(bar(B_DQ_FULL));
        ++dqc;
      }
    }
  } else {
    // ------------------------------------------------- element-wise work
    const int w = (warp - 2) >> 2;                // key-column quarter
    const int row = ((warp & 3) << 5) + lane;     // TMEM lane = query in the tile
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + 32u * w;
    const uint32_t tDP = tmem + lane_base + 128u + 32u * w;
    const uint32_t tDQ = tmem + lane_base + 256u + 32u * w;
    const uint32_t tQ = tmem + lane_base + 384u;
    const uint32_t tDO = tmem + lane_base + 448u;
    const size_t hstride = (size_t)p.n_tiles * 128;
    uint32_t steps = 0, dqc = 0;
    bool ok = true;
    for (uint32_t cons = 0; ok;) {
      const uint32_t sl = cons % kItemSlots;
      if (!__all_sync(0xffffffffu, mbar_wait(bar(B_ITEM_FULL + sl), (cons / kItemSlots) & 1, ab, 47))) {
        ok = false;
        break;
      }
      const int idx = item_slot[sl];
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_ITEM_EMPTY + sl));
      ++cons;
      if (idx >= n_items) break;
      const Item it = decode(p, idx);
      const int64_t q = (int64_t)it.i * 128 + row;
      const bool q_ok = q < p.S;
      const int32_t seg_q = q_ok ? (p.seg ? p.seg[(size_t)it.b * p.S + q] : 0) : -1;
      const size_t lrow = ((size_t)it.b * p.H + it.h) * hstride + (size_t)q;
      const float L2 = p.lse2[lrow];
      const float Dq = p.dpad[lrow];
      int n = 0;
      if (first_rel(p, it) >= 0) {
        // this quarter's 32 values of the row of Q~_i and of dO_i -> 16 columns each
        uint32_t qa[16], da[16];
        if (q_ok) {
          const size_t off = (((size_t)it.b * p.S + q) * p.H + it.h) * kD + 32 * w;
          const uint4* qs4 = reinterpret_cast<const uint4*>(p.q_rot + off);
          const uint4* ds4 = reinterpret_cast<const uint4*>(p.d_o + off);
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint4 a = qs4[c], d = ds4[c];
            qa[4 * c] = a.x; qa[4 * c + 1] = a.y; qa[4 * c + 2] = a.z; qa[4 * c + 3] = a.w;
            da[4 * c] = d.x; da[4 * c + 1] = d.y; da[4 * c + 2] = d.z; da[4 * c + 3] = d.w;
          }
        } else {
#pragma unroll
          for (int c = 0; c < 16; ++c) qa[c] = da[c] = 0u;
        }
        tmem_st16(tQ + 16 * w, qa);
        tmem_st16(tDO + 16 * w, da);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_Q_READY));
      }
      for (int j = it.lo; j <= it.hi; ++j) {
        if (!rel(p, it, j)) continue;
        const int64_t k0 = (int64_t)j * 128 + 32 * w;  // first key column of this quarter
        bool partial = (p.causal && j == it.i) || ((int64_t)(j + 1) * 128 > p.S) ||
                       ((int64_t)(it.i + 1) * 128 > p.S);
        if (p.seg) {
          const size_t kj = (size_t)it.b * p.n_tiles + j;
          const int32_t a0 = p.ktmin[kj], a1 = p.ktmax[kj];
          partial |= !(it.qmin >= 0 && it.qmin == it.qmax && a0 == it.qmin && a1 == it.qmin);
        }
        uint32_t mw = 0xffffffffu;
        if (partial) {
          // keep key k = k0 + c iff k < S, same segment, and k <= q when causal
          int hi = 32;  // exclusive
          if (p.causal) {
            const int64_t d = q - k0 + 1;
            hi = d < 0 ? 0 : (d > 32 ? 32 : (int)d);
          }
          const int64_t kv = p.S - k0;
          const int kvalid = kv > 32 ? 32 : (kv < 0 ? 0 : (int)kv);  // columns inside the row
          if (kvalid < hi) hi = kvalid;
          if (seg_q < 0) hi = 0;
          uint32_t bits = bit_range(0, hi);
          if (p.seg) {  // lane c loads the id of key column k0 + c
            const int32_t kid = lane < kvalid ? __ldg(p.kseg + (size_t)it.b * p.S + k0 + lane) : INT_MIN;
            bits &= warp_segment_bits(kid, seg_q);
          }
          mw = bits;
        }
        // ---- S -> registers; P = exp2(S * scale*log2e - LSE2[q]) ----
        if (!__all_sync(0xffffffffu, mbar_wait(bar(B_S_FULL), steps & 1, ab, 60 + w))) { ok = false; break; }
        tc_fence_after();
        uint32_t r[32];
        tmem_ld32(tS, r);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_S_READ));
        float pr[32];
        if (partial) {
#pragma unroll
          for (int c = 0; c < 32; ++c)
            pr[c] = ((mw >> c) & 1u) ? fast_exp2(fmaf(__uint_as_float(r[c]), p.scale_log2, -L2)) : 0.f;
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) pr[c] = fast_exp2(fmaf(__uint_as_float(r[c]), p.scale_log2, -L2));
        }
        // ---- dS = P o (dP - D[q]) back into tensor memory over dP ----
        if (!__all_sync(0xffffffffu, mbar_wait(bar(B_DP_FULL), steps & 1, ab, 62 + w))) { ok = false; break; }
        tc_fence_after();
        tmem_ld32(tDP, r);
        tmem_wait_ld();
        {
          uint32_t pk[16];
#pragma unroll
          for (int u = 0; u < 16; ++u)
            pk[u] = pack_bf16(pr[2 * u] * (__uint_as_float(r[2 * u]) - Dq),
                              pr[2 * u + 1] * (__uint_as_float(r[2 * u + 1]) - Dq));
          tmem_st16(tDP, pk);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_DS_FULL));
        ++steps;
        ++n;
      }
      if (!ok) break;
      // ---- dq epilogue (this quarter's 32 columns): scale, inverse rotation, bf16 ----
      __nv_bfloat16* dqrow = p.dq + (((size_t)it.b * p.S + (q_ok ? q : 0)) * p.H + it.h) * kD + 32 * w;
      if (n == 0) {
        if (q_ok) {
          const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
          for (int c = 0; c < 4; ++c) reinterpret_cast<uint4*>(dqrow)[c] = z;
        }
        continue;
      }
      if (!__all_sync(0xffffffffu, mbar_wait(bar(B_DQ_FULL), dqc & 1, ab, 64 + w))) { ok = false; break; }
      ++dqc;
      tc_fence_after();
      uint32_t r[32];
      tmem_ld32(tDQ, r);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_DQ_EMPTY));
      uint32_t out[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        float a = __uint_as_float(r[2 * u]) * p.scale, b = __uint_as_float(r[2 * u + 1]) * p.scale;
        if (p.rotate) {
          float c, s;
          rope_cos_sin_fast(q, freq[16 * w + u], &c, &s);
          const float a2 = a * c + b * s, b2 = b * c - a * s;
          a = a2;
          b = b2;
        }
        out[u] = pack_bf16(a, b);
      }
      if (q_ok) {
#pragma unroll
        for (int c = 0; c < 4; ++c)
          reinterpret_cast<uint4*>(dqrow)[c] =
              make_uint4(out[4 * c], out[4 * c + 1], out[4 * c + 2], out[4 * c + 3]);
      }
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
      for (uint32_t n = (k_issued > kKStages ? k_issued - kKStages : 0); n < k_issued; ++n)
        drain_wait(bar(B_K_FULL + n % kKStages), (n / kKStages) & 1);
      for (uint32_t n = (v_issued > kVStages ? v_issued - kVStages : 0); n < v_issued; ++n)
        drain_wait(bar(B_V_FULL + n % kVStages), (n / kVStages) & 1);
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

cudaError_t launch_sm100_bwd_dq(const Problem& pb, const Workspace& ws, const void* v,
                                const void* d_o, void* dq, cudaStream_t st) {
  CUtensorMap tk, tv;
  if (!make_qkv_map(&tk, ws.k_rot, pb.B, pb.S, pb.H, pb.D) ||
      !make_qkv_map(&tv, v, pb.B, pb.S, pb.H, pb.D))
    return cudaErrorInvalidValue;
  DqParams p{};
  p.q_rot = static_cast<const __nv_bfloat16*>(ws.q_rot);
  p.d_o = static_cast<const __nv_bfloat16*>(d_o);
  p.seg = pb.seg;
  p.kseg = pb.kseg;
  p.tmin = ws.tile_min;
  p.tmax = ws.tile_max;
  p.ktmin = ws.ktile_min;
  p.ktmax = ws.ktile_max;
  p.q_lo = ws.q_lo;
  p.lse2 = ws.lse2_pad;
  p.dpad = ws.delta_pad;
  p.dq = static_cast<__nv_bfloat16*>(dq);
  p.status = ws.status;
  p.S = pb.S;
  p.H = (int)pb.H;
  p.B = (int)pb.B;
  p.n_tiles = (int)pb.n_tiles;
  p.scale = pb.scale;
  p.scale_log2 = pb.scale * 1.4426950408889634f;
  p.causal = pb.causal;
  p.rotate = pb.theta > 0.0;
  p.log2_theta = p.rotate ? log2(pb.theta) : 0.0;
  const int64_t n_items = pb.B * pb.H * pb.n_tiles;
  if (n_items == 0) return cudaSuccess;
  static std::once_flag attr_once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(attr_once, [] {
    attr_err = cudaFuncSetAttribute(attn_bwd_dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)kSmemBytes);
  });
  if (attr_err != cudaSuccess) return attr_err;
  const int grid = (int)(n_items < sm_count() ? n_items : sm_count());
  attn_bwd_dq_kernel<<<grid, kThreads, kSmemBytes, st>>>(tk, tv, p);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace lwm
