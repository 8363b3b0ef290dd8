// Backward attention in one pass: dK, dV and dQ on the 5th-generation tensor
// cores (sm_100a), bf16, D=128.
//
// Gradients of sum(O * dO) for exact causal attention with a packing mask
// (LWM research note, "训练方法": training through the layer, Masked Sequence
// Packing).  P is recomputed from the saved LSE, as in the FlashAttention
// entry of the paper card's references.  Per (query tile i, key tile j):
//   S^T  = K~_j Q~_i^T            P^T  = exp(S^T * scale - LSE_i)
//   dP^T = V_j dO_i^T             dS^T = P^T o (dP^T - D_i),  D_i = dO_i . O_i
//   dV_j += P^T dO_i              dK~_j += dS^T Q~_i
//   dQ~_i += dS K~_j              (partial over key tile j)
// Every exponential and every product of the pair is computed once.
//
// One persistent CTA per SM owns a key tile j (128 keys) of one (b, h) and
// walks the query tiles i that may attend to it; dK_j and dV_j accumulate in
// tensor memory for the whole walk.  The dQ~_i partial of each step is
// computed in two 64-column halves; dedicated reducer warps read each half
// out of tensor memory and add it into an fp32 accumulator in global memory
// with vector reductions (performed in L2), so the element-wise warps never
// stall behind the reduction queue themselves; a short kernel then scales
// the accumulator, applies the inverse rotation and writes dq.  Roles (704
// threads):
//   warp 0      TMA producer: K_j (un-rotated: the element-wise warps apply
//               RoPE to it in shared memory), V_j once per item; per step Q~_i
//               with the tile's LSE*log2(e) and D (2-stage ring) and dO_i
//               (2-stage ring).
//   warp 1      MMA issuer (one thread); the whole warp allocates and frees
//               the tensor memory.
//   warps 4-19  element-wise work, four groups of four warps (one per TMEM
//               lane quarter, warp % 4) on 32 columns each: P^T (bf16) into
//               tensor memory, dS into a shared-memory tile, then the dK/dV
//               epilogue (bf16 blocks staged in the then idle dS tile and
//               sent by tensor stores).
//   warps 2, 3, 20, 21  dQ reducers, one per TMEM lane quarter.
// TMEM columns:
//   X  [0,128)    S^T(i), then dP^T(i) once S^T(i) is in registers
//   P  [128,192)  P^T(i), bf16 pairs (A operand of dV)
//   R  [192,256)  one 64-column half of the dQ~(i) partial (lanes = queries)
//   dV [256,384), dK [384,512)
// dS lives only in the shared tile: K-major it is the A operand of dK, MN-
// major the A operand of both dQ halves.
// MMA issue order per step:
//   dP^T(i) once S^T(i) is read | dQ(i-1) second half once R is read |
//   dV(i) after P(i) | S^T(i+1) once dP^T(i) is read | dK(i) after dS(i) |
//   dQ(i) first half once R is read
#include <cuda.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace lwm {

bool make_qkv_map(CUtensorMap* map, const void* ptr, int64_t B, int64_t S, int64_t H, int64_t D);
bool make_bf16_store_map(CUtensorMap* map, const void* ptr, int64_t B, int64_t S, int64_t H,
                         int64_t D);
int sm_count();

namespace {

using namespace sm100;

constexpr int kD = 128;
constexpr int kThreads = 704;   // TMA, MMA, 4 dQ reducer warps, 16 element-wise warps
constexpr int kEW = 512;        // element-wise threads
constexpr int kReducers = 4;    // dQ reducer warps, one per TMEM lane quarter
constexpr uint32_t kTileBytes = 128 * kD * 2;
constexpr uint32_t kBoxBytes = kTileBytes / 2;

// Tiles from the first 1024-byte boundary of dynamic shared memory (128-byte
// swizzle atoms):
constexpr uint32_t OFF_K = 0;
constexpr uint32_t OFF_V = OFF_K + kTileBytes;
constexpr uint32_t OFF_Q = OFF_V + kTileBytes;       // 2 stages
constexpr uint32_t OFF_DO = OFF_Q + 2 * kTileBytes;  // 2 stages
constexpr uint32_t OFF_DS = OFF_DO + 2 * kTileBytes; // dS: rows = keys, 128-byte swizzle
constexpr uint32_t kTilesBytes = OFF_DS + kTileBytes;  // 224 KB
// Small region after the tiles (16-byte aligned):
constexpr uint32_t SOFF_BAR = 0;                       // mbarriers
constexpr uint32_t SOFF_MISC = 256;                    // TMEM base, abort flag, item slots
constexpr uint32_t SOFF_LD = 320;                      // 2 stages x (LSE2[128], D[128]) fp32
constexpr uint32_t kLdStageBytes = 2 * 128 * 4;
constexpr uint32_t SOFF_FREQ = SOFF_LD + 2 * kLdStageBytes;  // 64 RoPE frequencies, fp64
constexpr uint32_t kSmallBytes = SOFF_FREQ + (kD / 2) * 8;
constexpr uint32_t kSmemBytes = 232448;                // the sm_100 per-block maximum
static_assert(kTilesBytes + kSmallBytes <= kSmemBytes, "shared memory layout");

enum : uint32_t {
  B_KV_FULL = 0, B_KV_EMPTY = 1,
  B_Q_FULL = 2,    // 2 stages
  B_Q_EMPTY = 4,   // 2 stages
  B_DO_FULL = 6,   // 2 stages
  B_DO_EMPTY = 8,  // 2 stages
  B_S_FULL = 10, B_S_READ = 11, B_DP_FULL = 12, B_DP_READ = 13, B_P_FULL = 14, B_DS_FULL = 15,
  B_DQA_FULL = 16, B_DKV_FULL = 17, B_DKV_EMPTY = 18, B_FIN = 19,
  B_ITEM_FULL = 20,   // 4 slots
  B_ITEM_EMPTY = 24,  // 4 slots
  B_K_ROT = 28,       // the element-wise warps rotated K~_j in place
  B_DQB_FULL = 29,    // second dQ half done: R holds it, and the dS tile is free
  B_R_EMPTY = 30,     // the reducer warps read R
  B_STG_FREE = 31,    // every element-wise warp's epilogue stores have read the dS tile
  B_COUNT = 32
};
static_assert(B_COUNT * 8 <= SOFF_MISC, "barrier slots");
constexpr uint32_t kItemSlots = 4;
constexpr uint32_t kEWWarps = kEW / 32;  // element-wise barriers take one arrival per warp

struct FusedParams {
  const int32_t* seg;    // query segment ids [B, S] or null
  const int32_t* kseg;   // key segment ids (seg unless a block pair)
  const int32_t* tmin;   // query tile bounds
  const int32_t* tmax;
  const int32_t* ktmin;  // key tile bounds
  const int32_t* ktmax;
  const int32_t* k_hi;
  const float* lse2;     // [B, H, nT*128]: LSE * log2(e), +inf where the row has no keys
  const float* dpad;     // [B, H, nT*128]: dot(dO, O), 0 past the end
  float* dq_acc;         // [B*H, nT, 32, 128, 4]: unscaled dQ~ partial sums (zeroed)
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  float* dk32;           // non-null: dK, dV written in fp32 here instead (block partials)
  float* dv32;
  DeviceStatus* status;
  int64_t S;
  int H, B, n_tiles;
  float scale, scale_log2;
  int causal, rotate;    // rotate: RoPE on (inverse rotation of dK, dQ)
  int rot_k;             // K_j arrives un-rotated: RoPE it in shared memory
  int out_v8;            // the dK, dV outputs are 32-byte aligned: 256-bit row stores
  int tma_out;           // bf16 dK, dV leave by tensor stores through the dS tile
  double log2_theta;
};

struct Item {
  int b, h, j;
  int lo, hi;          // query tile range
  int32_t kmin, kmax;  // key tile id range
};

__device__ __forceinline__ bool meet(int32_t a0, int32_t a1, int32_t b0, int32_t b1) {
  return a1 >= 0 && b1 >= 0 && a0 <= b1 && b0 <= a1;
}

__device__ __forceinline__ Item decode(const FusedParams& p, int idx) {
  Item it;
  const int bh = idx / p.n_tiles;
  it.j = idx % p.n_tiles;  // ascending key tile = most query tiles first (causal)
  it.b = bh / p.H;
  it.h = bh % p.H;
  it.lo = p.causal ? it.j : 0;
  it.hi = p.n_tiles - 1;
  it.kmin = 0;
  it.kmax = 0;
  if (p.seg) {
    const size_t kj = (size_t)it.b * p.n_tiles + it.j;
    it.hi = p.k_hi[kj];
    it.kmin = p.ktmin[kj];
    it.kmax = p.ktmax[kj];
  }
  return it;
}

__device__ __forceinline__ bool rel(const FusedParams& p, const Item& it, int i) {
  if (i < it.lo || i > it.hi) return false;
  if (!p.seg) return true;
  const size_t qi = (size_t)it.b * p.n_tiles + i;
  return meet(it.kmin, it.kmax, p.tmin[qi], p.tmax[qi]);
}

__device__ __forceinline__ int next_rel(const FusedParams& p, const Item& it, int i) {
  for (++i; i <= it.hi; ++i)
    if (rel(p, it, i)) return i;
  return -1;
}

__device__ __forceinline__ int first_rel(const FusedParams& p, const Item& it) {
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
attn_bwd_fused_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                      const __grid_constant__ CUtensorMap tm_dk, const __grid_constant__ CUtensorMap tm_dv,
                      const FusedParams p) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  const uint32_t small = base + kTilesBytes;
  if (small + kSmallBytes > raw + kSmemBytes) {  // same outcome in every thread
    if (threadIdx.x == 0) report_status(p.status, LWM_ERR_UNSUPPORTED, 0);
    return;
  }
  uint8_t* small_ptr = smem_raw + (small - raw);
  const uint32_t bar0 = small + SOFF_BAR;
  auto bar = [&](uint32_t slot) { return bar0 + 8u * slot; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(small_ptr + SOFF_MISC + 8);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(small_ptr + SOFF_MISC);
  const float* ld_smem = reinterpret_cast<const float*>(small_ptr + SOFF_LD);
  double* freq = reinterpret_cast<double*>(small_ptr + SOFF_FREQ);
  // work items come from a global counter (greedy, in cost order): the TMA
  // thread takes one and publishes it to the CTA through a 4-slot ring
  volatile int* item_slot = reinterpret_cast<volatile int*>(small_ptr + SOFF_MISC + 16);
  int* item_counter = &p.status->item_counter[3];
  const Abort ab{abort_flag, p.status};
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_items = p.B * p.H * p.n_tiles;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(bar(B_KV_FULL), 1);
    mbar_init(bar(B_KV_EMPTY), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(B_Q_FULL + s), 1);
      mbar_init(bar(B_Q_EMPTY + s), 1);
      mbar_init(bar(B_DO_FULL + s), 1);
      mbar_init(bar(B_DO_EMPTY + s), 1);
    }
    mbar_init(bar(B_S_FULL), 1);
    mbar_init(bar(B_S_READ), kEWWarps);
    mbar_init(bar(B_DP_FULL), 1);
    mbar_init(bar(B_DP_READ), kEWWarps);
    mbar_init(bar(B_P_FULL), kEWWarps);
    mbar_init(bar(B_DS_FULL), kEWWarps);
    mbar_init(bar(B_DQA_FULL), 1);
    mbar_init(bar(B_DQB_FULL), 1);
    mbar_init(bar(B_R_EMPTY), kReducers);
    mbar_init(bar(B_DKV_FULL), 1);
    mbar_init(bar(B_DKV_EMPTY), kEWWarps);
    mbar_init(bar(B_FIN), 1);
    for (uint32_t sl = 0; sl < kItemSlots; ++sl) {
      mbar_init(bar(B_ITEM_FULL + sl), 1);
      mbar_init(bar(B_ITEM_EMPTY + sl), 1 + kEWWarps + kReducers);
    }
    mbar_init(bar(B_K_ROT), kEWWarps);
    mbar_init(bar(B_STG_FREE), kEWWarps);
    fence_mbar_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_do);
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
  uint32_t q_issued = 0, do_issued = 0, kv_issued = 0;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA
    if (lane == 0) {
      uint32_t q_it = 0, do_it = 0;
      int items = 0;
      bool ok = true;
      const size_t hstride = (size_t)p.n_tiles * 128;
      for (uint32_t pub = 0; ok; ++items) {
        const uint32_t sl = pub % kItemSlots;
        if (pub >= kItemSlots &&
            !mbar_wait(bar(B_ITEM_EMPTY + sl), ((pub / kItemSlots) - 1) & 1, ab, 70)) {
          ok = false;
          break;
        }
        const int idx = atomicAdd(item_counter, 1);
        item_slot[sl] = idx;
        mbar_arrive(bar(B_ITEM_FULL + sl));
        ++pub;
        if (idx >= n_items) break;
        const Item it = decode(p, idx);
        int i = first_rel(p, it);
        if (i < 0) continue;  // nothing to load: the element-wise warps write zeros
        if (kv_issued > 0 && !mbar_wait(bar(B_KV_EMPTY), (kv_issued - 1) & 1, ab, 71)) { ok = false; break; }
        mbar_expect_tx(bar(B_KV_FULL), 2 * kTileBytes);
        tma_load_4d(base + OFF_K, &tm_k, bar(B_KV_FULL), 0, it.h, it.j * 128, it.b);
        tma_load_4d(base + OFF_K + kBoxBytes, &tm_k, bar(B_KV_FULL), 64, it.h, it.j * 128, it.b);
        tma_load_4d(base + OFF_V, &tm_v, bar(B_KV_FULL), 0, it.h, it.j * 128, it.b);
        tma_load_4d(base + OFF_V + kBoxBytes, &tm_v, bar(B_KV_FULL), 64, it.h, it.j * 128, it.b);
        ++kv_issued;
        const float* lse2 = p.lse2 + ((size_t)it.b * p.H + it.h) * hstride;
        const float* dpad = p.dpad + ((size_t)it.b * p.H + it.h) * hstride;
        for (; i >= 0; i = next_rel(p, it, i)) {
          const uint32_t s = q_it & 1;
          if (!mbar_wait(bar(B_Q_EMPTY + s), ((q_it >> 1) & 1) ^ 1, ab, 72)) { ok = false; break; }
          mbar_expect_tx(bar(B_Q_FULL + s), kTileBytes + kLdStageBytes);
          const uint32_t dq = base + OFF_Q + s * kTileBytes;
          tma_load_4d(dq, &tm_q, bar(B_Q_FULL + s), 0, it.h, i * 128, it.b);
          tma_load_4d(dq + kBoxBytes, &tm_q, bar(B_Q_FULL + s), 64, it.h, i * 128, it.b);
          const uint32_t ld = small + SOFF_LD + s * kLdStageBytes;
          bulk_load(ld, lse2 + (size_t)i * 128, 512, bar(B_Q_FULL + s));
          bulk_load(ld + 512, dpad + (size_t)i * 128, 512, bar(B_Q_FULL + s));
          q_issued = ++q_it;
          const uint32_t t = do_it & 1;
          if (!mbar_wait(bar(B_DO_EMPTY + t), ((do_it >> 1) & 1) ^ 1, ab, 73)) { ok = false; break; }
          mbar_expect_tx(bar(B_DO_FULL + t), kTileBytes);
          const uint32_t dd = base + OFF_DO + t * kTileBytes;
          tma_load_4d(dd, &tm_do, bar(B_DO_FULL + t), 0, it.h, i * 128, it.b);
          tma_load_4d(dd + kBoxBytes, &tm_do, bar(B_DO_FULL + t), 64, it.h, i * 128, it.b);
          do_issued = ++do_it;
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA
    if (lane == 0) {
      constexpr uint32_t kIdKK = idesc_bf16(128, 128, 0, 0);   // K-major x K-major
      constexpr uint32_t kIdKM = idesc_bf16(128, 128, 0, 1);   // K-major (TMEM or smem) x MN-major
      constexpr uint32_t kIdMM = idesc_bf16(128, 64, 1, 1);    // MN-major x MN-major, N = 64
      const uint32_t sK = base + OFF_K, sV = base + OFF_V;
      const uint32_t tX = tmem, tP = tmem + 128, tR = tmem + 192, tDV = tmem + 256, tDK = tmem + 384;
      uint32_t q_it = 0, do_it = 0, steps = 0, dkv = 0, kv_items = 0, halves = 0;
      bool ok = true;
      const uint64_t dK = kmajor_desc(sK), dV = kmajor_desc(sV);
      const uint64_t dDSk = kmajor_desc(base + OFF_DS), dDSmn = mnmajor_desc(base + OFF_DS);
      auto sq_of = [&](uint32_t n) { return base + OFF_Q + (n & 1) * kTileBytes; };
      auto sdo_of = [&](uint32_t n) { return base + OFF_DO + (n & 1) * kTileBytes; };
      auto issue_s = [&](uint32_t n) -> bool {
        if (!mbar_wait(bar(B_Q_FULL + (n & 1)), (n >> 1) & 1, ab, 74)) return false;
        tc_fence_after();
        mma_kk128(tX, dK, kmajor_desc(sq_of(n)), kIdKK, 0u);
        mma_commit(bar(B_S_FULL));
        return true;
      };
      // half h of dQ~(i) = dS(i) K~ (D columns 64h..64h+63) into R, once the
      // reducer warps have read the previous half out of it
      auto issue_half = [&](uint32_t h) -> bool {
        if (halves > 0 && !mbar_wait(bar(B_R_EMPTY), (halves - 1) & 1, ab, 110)) return false;
        tc_fence_after();
        mma_mm128(tR, dDSmn, mnmajor_desc(sK + h * kBoxBytes), kIdMM, 0u);
        mma_commit(bar(h ? B_DQB_FULL : B_DQA_FULL));
        ++halves;
        return true;
      };
      for (uint32_t cons = 0; ok;) {
        const uint32_t sl = cons % kItemSlots;
        if (!mbar_wait(bar(B_ITEM_FULL + sl), (cons / kItemSlots) & 1, ab, 75)) { ok = false; break; }
        const int idx = item_slot[sl];
        mbar_arrive(bar(B_ITEM_EMPTY + sl));
        ++cons;
        if (idx >= n_items) break;
        const Item it = decode(p, idx);
        int i = first_rel(p, it);
        if (i < 0) continue;
        if (!mbar_wait(bar(B_KV_FULL), kv_items & 1, ab, 76)) { ok = false; break; }
        // K~_j arrives un-rotated: the element-wise warps rotate it in place
        if (p.rot_k && !mbar_wait(bar(B_K_ROT), kv_items & 1, ab, 108)) { ok = false; break; }
        ++kv_items;
        tc_fence_after();
        // X is free: the previous item's last dP^T was read before its dK
        if (!issue_s(q_it)) { ok = false; break; }
        bool first = true, pend_b = false;
        while (i >= 0) {
          // dP^T(i) into X once S^T(i) is in registers
          if (!mbar_wait(bar(B_S_READ), steps & 1, ab, 77)) { ok = false; break; }
          if (!mbar_wait(bar(B_DO_FULL + (do_it & 1)), (do_it >> 1) & 1, ab, 78)) { ok = false; break; }
          tc_fence_after();
          mma_kk128(tX, dV, kmajor_desc(sdo_of(do_it)), kIdKK, 0u);
          mma_commit(bar(B_DP_FULL));
          // the previous step's second dQ half, behind dP^T(i) in the pipe
          if (pend_b && !issue_half(1)) { ok = false; break; }
          pend_b = false;
          // dV(i) += P^T dO  (P^T from TMEM)
          if (first && dkv > 0 && !mbar_wait(bar(B_DKV_EMPTY), (dkv - 1) & 1, ab, 79)) { ok = false; break; }
          if (!mbar_wait(bar(B_P_FULL), steps & 1, ab, 80)) { ok = false; break; }
          tc_fence_after();
          mma_tm128<false>(tDV, tP, mnmajor_desc(sdo_of(do_it)), kIdKM, first ? 0u : 1u);
          mma_commit(bar(B_DO_EMPTY + (do_it & 1)));
          ++do_it;
          // S^T(next) into X once dP^T(i) is in registers
          const int inext = next_rel(p, it, i);
          if (!mbar_wait(bar(B_DP_READ), steps & 1, ab, 81)) { ok = false; break; }
          if (inext >= 0 && !issue_s(q_it + 1)) { ok = false; break; }
          // dK(i) += dS^T Q~ (dS^T: the shared dS tile read K-major), then the
          // first dQ half (the same tile read MN-major)
          if (!mbar_wait(bar(B_DS_FULL), steps & 1, ab, 82)) { ok = false; break; }
          tc_fence_after();
          mma_km128(tDK, dDSk, mnmajor_desc(sq_of(q_it)), kIdKM, first ? 0u : 1u);
          mma_commit(bar(B_Q_EMPTY + (q_it & 1)));
          if (!issue_half(0)) { ok = false; break; }
          pend_b = true;
          ++q_it;
          ++steps;
          first = false;
          i = inext;
        }
        if (!ok) break;
        if (pend_b && !issue_half(1)) { ok = false; break; }
        mma_commit(bar(B_DKV_FULL));
        ++dkv;
        mma_commit(bar(B_KV_EMPTY));  // K~_j (read by the last dQ half) and V_j are free
      }
    }
  } else if (warp >= 4 && warp < 4 + kEWWarps) {
    // ------------------------------------------------- element-wise work
    const int w = (warp - 4) >> 2;                // column quarter
    const int row = ((warp & 3) << 5) + lane;     // TMEM lane = key
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tX = tmem + lane_base + 32u * w;
    const uint32_t tP = tmem + lane_base + 128u + 16u * w;
    const uint32_t tDV = tmem + lane_base + 256u + 32u * w;
    const uint32_t tDK = tmem + lane_base + 384u + 32u * w;
    // this thread's 64 bytes of the dS tile: key row `row`, query columns
    // 32w..32w+31 = 16-byte chunks 4(w&1)..4(w&1)+3 of box w>>1, swizzled
    const uint32_t sDSrow = base + OFF_DS + (uint32_t)(w >> 1) * kBoxBytes + (uint32_t)row * 128u;
    const uint32_t chunk0 = (uint32_t)(w & 1) * 4u, swz = (uint32_t)row & 7u;
    uint32_t steps = 0, dkv = 0, kv_items = 0;
    bool ok = true;
    for (uint32_t cons = 0; ok;) {
      const uint32_t sl = cons % kItemSlots;
      if (!__all_sync(0xffffffffu, mbar_wait(bar(B_ITEM_FULL + sl), (cons / kItemSlots) & 1, ab, 83))) {
        ok = false;
        break;
      }
      const int idx = item_slot[sl];
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_ITEM_EMPTY + sl));
      ++cons;
      if (idx >= n_items) break;
      const Item it = decode(p, idx);
      const int64_t key = (int64_t)it.j * 128 + row;
      const bool key_ok = key < p.S;
      const int32_t seg_k = key_ok ? (p.seg ? p.kseg[(size_t)it.b * p.S + key] : 0) : -1;
      int n = 0;
      const bool has_tiles = first_rel(p, it) >= 0;
      if (p.tma_out && has_tiles && dkv > 0) {
        // this item writes dS tiles: the dK/dV tensor stores of the previous
        // item with tiles (dkv - 1), staged all over the tile, must have read
        // it in every warp
        if (lane == 0) bulk_wait_read0();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_STG_FREE));
        if (!__all_sync(0xffffffffu, mbar_wait(bar(B_STG_FREE), (dkv - 1) & 1, ab, 116 + w))) {
          ok = false;
          break;
        }
      }
      if (p.rot_k && has_tiles) {
        // RoPE on this thread's 32 columns of key row `row` of K~_j, in place
        // in shared memory (the producer loaded it un-rotated): pair (2i,
        // 2i+1) turns by key * w_i, the angle reduced in fp64 and cos/sin from
        // the fast approximation (absolute error below 1e-6, far under the
        // bf16 rounding of the result)
        if (!__all_sync(0xffffffffu, mbar_wait(bar(B_KV_FULL), kv_items & 1, ab, 109))) {
          ok = false;
          break;
        }
        const uint32_t krow = base + OFF_K + (uint32_t)(w >> 1) * kBoxBytes + (uint32_t)row * 128u;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          const uint32_t a = krow + (((chunk0 + (uint32_t)c) ^ swz) << 4);
          uint32_t v4[4];
          asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(v4[0]), "=r"(v4[1]), "=r"(v4[2]), "=r"(v4[3]) : "r"(a));
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            float cs, sn;
            rope_cos_sin_fast(key, freq[16 * w + 4 * c + u], &cs, &sn);
            const float x0 = __uint_as_float(v4[u] << 16), x1 = __uint_as_float(v4[u] & 0xffff0000u);
            v4[u] = pack_bf16(x0 * cs - x1 * sn, x0 * sn + x1 * cs);
          }
          st_shared_v4(a, v4[0], v4[1], v4[2], v4[3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_K_ROT));
        ++kv_items;
      }
      // segment bounds of query tile i, loaded one tile ahead so that their
      // latency stays off the element-wise path
      const size_t qi0 = (size_t)it.b * p.n_tiles;
      int32_t nb0 = 0, nb1 = 0;
      if (p.seg && it.lo <= it.hi) {
        nb0 = p.tmin[qi0 + it.lo];
        nb1 = p.tmax[qi0 + it.lo];
      }
      for (int i = it.lo; i <= it.hi; ++i) {
        const int32_t a0 = nb0, a1 = nb1;
        if (p.seg && i < it.hi) {
          nb0 = p.tmin[qi0 + i + 1];
          nb1 = p.tmax[qi0 + i + 1];
        }
        // rel(p, it, i) with the bounds already loaded
        if (p.seg && !meet(it.kmin, it.kmax, a0, a1)) continue;
        const int64_t q0 = (int64_t)i * 128 + 32 * w;  // first query column of this quarter
        bool partial = (p.causal && i == it.j) || ((int64_t)(i + 1) * 128 > p.S) ||
                       ((int64_t)(it.j + 1) * 128 > p.S);
        if (p.seg)
          partial |= !(it.kmin >= 0 && it.kmin == it.kmax && a0 == it.kmin && a1 == it.kmin);
        uint32_t mw = 0xffffffffu;
        if (partial) {
          // keep query q = q0 + c iff q < S, same segment, and q >= key when causal
          int lo = 0;
          if (p.causal) {
            const int64_t d = key - q0;
            lo = d < 0 ? 0 : (d > 32 ? 32 : (int)d);
          }
          const int64_t qv = p.S - q0;
          const int hi = qv > 32 ? 32 : (qv < 0 ? 0 : (int)qv);  // exclusive
          uint32_t bits = seg_k >= 0 ? bit_range(lo, hi) : 0u;
          if (p.seg) {  // lane c loads the id of query column q0 + c
            const int32_t qseg = lane < hi ? __ldg(p.seg + (size_t)it.b * p.S + q0 + lane) : INT_MIN;
            bits &= warp_segment_bits(qseg, seg_k);
          }
          mw = bits;
        }
        const uint32_t stage = steps & 1;
        const float* lse2 = ld_smem + stage * (kLdStageBytes / 4) + 32 * w;
        const float* dsum = lse2 + 128;
        // ---- S^T -> registers; P^T = exp2(S^T * scale*log2e - LSE2[q]) ----
        if (!__all_sync(0xffffffffu, mbar_wait(bar(B_S_FULL), steps & 1, ab, 84 + w) &&
                                         mbar_wait(bar(B_Q_FULL + stage), (steps >> 1) & 1, ab, 88 + w))) {
          ok = false;
          break;
        }
        tc_fence_after();
        float pr[32];
        {
          uint32_t r[32];
          tmem_ld32(tX, r);
          tmem_wait_ld();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(B_S_READ));  // dP^T(i) may overwrite X now
          const float4* l4 = reinterpret_cast<const float4*>(lse2);
          if (partial) {
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const float4 L = l4[u];
              const float Ls[4] = {L.x, L.y, L.z, L.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int c = 4 * u + e;
                pr[c] = ((mw >> c) & 1u) ? fast_exp2(fmaf(__uint_as_float(r[c]), p.scale_log2, -Ls[e]))
                                         : 0.f;
              }
            }
          } else {
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const float4 L = l4[u];
              const float Ls[4] = {L.x, L.y, L.z, L.w};
#pragma unroll
              for (int e = 0; e < 4; ++e)
                pr[4 * u + e] = fast_exp2(fmaf(__uint_as_float(r[4 * u + e]), p.scale_log2, -Ls[e]));
            }
          }
        }
        // ---- P^T (bf16) into this warp's 16 columns of P (dV(i-1), which
        // read them, completed before S^T(i)) ----
        {
          uint32_t pk[16];
#pragma unroll
          for (int u = 0; u < 16; ++u) pk[u] = pack_bf16(pr[2 * u], pr[2 * u + 1]);
          tmem_st16(tP, pk);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_P_FULL));
        // ---- dS = P o (dP - D[q]): dP^T(i) read out of X as soon as it is
        // done (so S^T(i+1) can start), then dS into the shared tile (the A
        // operand of dK and of both dQ halves) once the second dQ half of the
        // previous step has read the tile ----
        if (!__all_sync(0xffffffffu, mbar_wait(bar(B_DP_FULL), steps & 1, ab, 96 + w))) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t ds[16];
        {
          const float4* d4 = reinterpret_cast<const float4*>(dsum);
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            uint32_t r[16];
            tmem_ld16(tX + 16u * hh, r);
            tmem_wait_ld();
            if (hh == 1) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(bar(B_DP_READ));  // S^T(i+1) may overwrite X now
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const float4 Dv = d4[4 * hh + u];
              const float* pp = pr + 16 * hh + 4 * u;
              ds[8 * hh + 2 * u] = pack_bf16(pp[0] * (__uint_as_float(r[4 * u]) - Dv.x),
                                             pp[1] * (__uint_as_float(r[4 * u + 1]) - Dv.y));
              ds[8 * hh + 2 * u + 1] = pack_bf16(pp[2] * (__uint_as_float(r[4 * u + 2]) - Dv.z),
                                                 pp[3] * (__uint_as_float(r[4 * u + 3]) - Dv.w));
            }
          }
        }
        // the shared dS tile is free once the previous step's second dQ half has read it
        if (!__all_sync(0xffffffffu, steps == 0 || mbar_wait(bar(B_DQB_FULL), (steps - 1) & 1, ab, 100 + w))) {
          ok = false;
          break;
        }
#pragma unroll
        for (int c = 0; c < 4; ++c)
          st_shared_v4(sDSrow + (((chunk0 + c) ^ swz) << 4), ds[4 * c], ds[4 * c + 1], ds[4 * c + 2],
                       ds[4 * c + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_DS_FULL));
        ++steps;
        ++n;
      }
      if (!ok) break;
      // ---- dK, dV epilogue for this key tile (this quarter's 32 columns) ----
      const size_t orow_off = (((size_t)it.b * p.S + (key_ok ? key : 0)) * p.H + it.h) * kD + 32 * w;
      if (n == 0) {
        if (key_ok) {
          const uint4 z = make_uint4(0, 0, 0, 0);
          if (p.dk32) {
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              reinterpret_cast<uint4*>(p.dk32 + orow_off)[c] = z;
              reinterpret_cast<uint4*>(p.dv32 + orow_off)[c] = z;
            }
          } else {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              reinterpret_cast<uint4*>(p.dk + orow_off)[c] = z;
              reinterpret_cast<uint4*>(p.dv + orow_off)[c] = z;
            }
          }
        }
        continue;
      }
      if (!__all_sync(0xffffffffu, mbar_wait(bar(B_DKV_FULL), dkv & 1, ab, 104 + w))) { ok = false; break; }
      ++dkv;
      tc_fence_after();
      // 32 fp32 values of a row out: bf16 pairs, or fp32 for block partials
      auto store_row = [&](__nv_bfloat16* dst16, float* dst32, const float (&x)[32]) {
        if (!key_ok) return;
        // Each lane writes its own row: the fewer store instructions, the
        // fewer passes the L1 makes over 32 rows, so 256-bit stores where the
        // outputs are 32-byte aligned
        if (dst32) {
          if (p.out_v8) {
#pragma unroll
            for (int c = 0; c < 4; ++c)
              st_global_v8(dst32 + 8 * c, __float_as_uint(x[8 * c]), __float_as_uint(x[8 * c + 1]),
                           __float_as_uint(x[8 * c + 2]), __float_as_uint(x[8 * c + 3]),
                           __float_as_uint(x[8 * c + 4]), __float_as_uint(x[8 * c + 5]),
                           __float_as_uint(x[8 * c + 6]), __float_as_uint(x[8 * c + 7]));
          } else {
#pragma unroll
            for (int c = 0; c < 8; ++c)
              reinterpret_cast<float4*>(dst32)[c] = make_float4(x[4 * c], x[4 * c + 1], x[4 * c + 2], x[4 * c + 3]);
          }
        } else {
          uint32_t pk[16];
#pragma unroll
          for (int u = 0; u < 16; ++u) pk[u] = pack_bf16(x[2 * u], x[2 * u + 1]);
          if (p.out_v8) {
            st_global_v8(dst16, pk[0], pk[1], pk[2], pk[3], pk[4], pk[5], pk[6], pk[7]);
            st_global_v8(dst16 + 16, pk[8], pk[9], pk[10], pk[11], pk[12], pk[13], pk[14], pk[15]);
          } else {
#pragma unroll
            for (int c = 0; c < 4; ++c)
              reinterpret_cast<uint4*>(dst16)[c] = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
          }
        }
      };
      // tensor stores: this warp's 32 keys x 32 columns in bf16 are staged
      // in its own dense 2 KB of the dS tile (rows of 64 bytes, 16-byte
      // chunk c of row r at slot c ^ ((r >> 1) & 3): the 64-byte swizzle,
      // conflict-free) and leave in one box per tensor
      const uint32_t stg = base + OFF_DS + (uint32_t)(warp - 4) * 2048u;
      const int krow0 = it.j * 128 + ((warp & 3) << 5);
      auto stage_row = [&](const float (&x)[32]) {
        uint32_t pk[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) pk[u] = pack_bf16(x[2 * u], x[2 * u + 1]);
#pragma unroll
        for (int c = 0; c < 4; ++c)
          st_shared_v4(stg + (uint32_t)lane * 64u + (uint32_t)((c ^ ((lane >> 1) & 3)) << 4), pk[4 * c],
                       pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        fence_proxy_async_smem();
        __syncwarp();
      };
      {
        uint32_t r[32];
        tmem_ld32(tDV, r);
        tmem_wait_ld();
        float x[32];
#pragma unroll
        for (int u = 0; u < 32; ++u) x[u] = __uint_as_float(r[u]);
        if (p.tma_out) {
          stage_row(x);
          if (lane == 0) {
            tma_store_4d(&tm_dv, stg, 32 * w, it.h, krow0, it.b);
            bulk_commit();
          }
        } else {
          store_row(p.dv + orow_off, p.dv32 ? p.dv32 + orow_off : nullptr, x);
        }
      }
      {
        uint32_t r[32];
        tmem_ld32(tDK, r);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_DKV_EMPTY));
        float x[32];
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          float a = __uint_as_float(r[2 * u]) * p.scale, b = __uint_as_float(r[2 * u + 1]) * p.scale;
          if (p.rotate) {
            float c, s;
            rope_cos_sin_fast(key, freq[16 * w + u], &c, &s);
            const float a2 = a * c + b * s, b2 = b * c - a * s;
            a = a2;
            b = b2;
          }
          x[2 * u] = a;
          x[2 * u + 1] = b;
        }
        if (p.tma_out) {
          if (lane == 0) bulk_wait_read0();  // dV's store has read the staging slots
          __syncwarp();
          stage_row(x);
          if (lane == 0) {
            tma_store_4d(&tm_dk, stg, 32 * w, it.h, krow0, it.b);
            bulk_commit();
          }
        } else {
          store_row(p.dk + orow_off, p.dk32 ? p.dk32 + orow_off : nullptr, x);
        }
      }
    }
    if (lane == 0) bulk_wait0();  // this warp's tensor stores have completed
  } else {
    // ------------------------------------------------------- dQ reducers
    // One warp per TMEM lane quarter (warps 2, 3, 20, 21).  Each half of a
    // step's dQ~ partial is read out of R (32 query rows x 64 columns per
    // warp), R is handed back to the MMA warp, and the half is added into the
    // accumulator tile with sixteen 512-byte vector reductions per warp while
    // the other roles go on.
    const int row = ((warp & 3) << 5) + lane;  // TMEM lane = query row of the tile
    const uint32_t tR = tmem + ((uint32_t)((warp & 3) * 32) << 16) + 192u;
    uint32_t steps = 0;
    bool ok = true;
    for (uint32_t cons = 0; ok;) {
      const uint32_t sl = cons % kItemSlots;
      if (!__all_sync(0xffffffffu, mbar_wait(bar(B_ITEM_FULL + sl), (cons / kItemSlots) & 1, ab, 111))) {
        ok = false;
        break;
      }
      const int idx = item_slot[sl];
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_ITEM_EMPTY + sl));
      ++cons;
      if (idx >= n_items) break;
      const Item it = decode(p, idx);
      float* acc_bh = p.dq_acc + ((size_t)it.b * p.H + it.h) * (size_t)p.n_tiles * (128 * kD);
      for (int i = first_rel(p, it); i >= 0 && ok; i = next_rel(p, it, i)) {
#pragma unroll 1
        for (int h = 0; h < 2; ++h) {
          if (!__all_sync(0xffffffffu, mbar_wait(bar(h ? B_DQB_FULL : B_DQA_FULL), steps & 1, ab, 112 + h))) {
            ok = false;
            break;
          }
          tc_fence_after();
          uint32_t ra[32], rb[32];
          tmem_ld32(tR, ra);
          tmem_ld32(tR + 32u, rb);
          tmem_wait_ld();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(B_R_EMPTY));
          // columns 64h..64h+63 = column groups 16h..16h+15 of [32][128][4]
          float* dst = acc_bh + (size_t)i * (128 * kD) + ((size_t)(16 * h) * 128 + row) * 4;
#pragma unroll
          for (int g = 0; g < 8; ++g)
            red_add_v4(dst + (size_t)g * 512, __uint_as_float(ra[4 * g]), __uint_as_float(ra[4 * g + 1]),
                       __uint_as_float(ra[4 * g + 2]), __uint_as_float(ra[4 * g + 3]));
#pragma unroll
          for (int g = 0; g < 8; ++g)
            red_add_v4(dst + (size_t)(8 + g) * 512, __uint_as_float(rb[4 * g]), __uint_as_float(rb[4 * g + 1]),
                       __uint_as_float(rb[4 * g + 2]), __uint_as_float(rb[4 * g + 3]));
        }
        ++steps;
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
      if (kv_issued > 0) drain_wait(bar(B_KV_FULL), (kv_issued - 1) & 1);
      for (uint32_t n = (q_issued > 2 ? q_issued - 2 : 0); n < q_issued; ++n)
        drain_wait(bar(B_Q_FULL + (n & 1)), (n >> 1) & 1);
      for (uint32_t n = (do_issued > 2 ? do_issued - 2 : 0); n < do_issued; ++n)
        drain_wait(bar(B_DO_FULL + (n & 1)), (n >> 1) & 1);
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// dq = R(p)^T (scale * dQ~) in bf16 (or fp32), from the fp32 accumulator:
// one CTA per half (64 rows) of a (b, h, query tile).  The half's 32 KB of
// the tile ([32 column groups][128 rows][4]: 32 runs of 1 KB) comes in with
// fully coalesced 16-byte loads and is transposed through shared memory
// (rows padded by 4 floats: conflict-free 16-byte stores); then each warp
// writes whole rows, lane l holding columns 4l..4l+3, so a row's 256 (or
// 512) bytes leave in one contiguous store.  Half tiles keep six CTAs on an
// SM, so that loads of some overlap the stores of others.
constexpr int kFinRow = kD + 4;  // padded shared-memory row, floats
constexpr int kFinRows = 64;     // rows per CTA
constexpr int kFinThreads = 256;
__global__ void __launch_bounds__(kFinThreads)
dq_finish_kernel(const float* __restrict__ acc, __nv_bfloat16* __restrict__ dq, float* __restrict__ dq32,
                 int64_t S, int H, int n_tiles, float scale, int rotate, double log2_theta) {
  extern __shared__ float tile[];  // [kFinRows][kFinRow]
  __shared__ double freq[kD / 2];
  if (threadIdx.x < kD / 2 && rotate) freq[threadIdx.x] = rope_freq(threadIdx.x, kD, log2_theta);
  const int64_t t_all = blockIdx.x >> 1;  // (b, h, query tile)
  const int half = blockIdx.x & 1;
  const float4* src = reinterpret_cast<const float4*>(acc + (size_t)t_all * (128 * kD)) + kFinRows * half;
#pragma unroll 8
  for (int k = 0; k < 32 * kFinRows / kFinThreads; ++k) {
    const int j = threadIdx.x + kFinThreads * k;  // column group j / 64, row j % 64 of the half
    *reinterpret_cast<float4*>(&tile[(j & (kFinRows - 1)) * kFinRow + (j / kFinRows) * 4]) =
        src[(j / kFinRows) * 128 + (j & (kFinRows - 1))];
  }
  __syncthreads();
  const int tile_i = (int)(t_all % n_tiles);
  const int64_t bh = t_all / n_tiles;
  const int64_t b = bh / H, h = bh % H;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int r = warp; r < kFinRows; r += kFinThreads / 32) {
    const int64_t q = (int64_t)tile_i * 128 + kFinRows * half + r;
    if (q >= S) break;
    const float4 v = *reinterpret_cast<const float4*>(&tile[r * kFinRow + 4 * lane]);
    float x[4] = {v.x * scale, v.y * scale, v.z * scale, v.w * scale};
    if (rotate) {
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        float c, sn;
        rope_cos_sin_fast(q, freq[2 * lane + u], &c, &sn);
        const float a = x[2 * u], bb = x[2 * u + 1];
        x[2 * u] = a * c + bb * sn;
        x[2 * u + 1] = bb * c - a * sn;
      }
    }
    const size_t off = (((size_t)b * S + q) * H + h) * kD + 4 * lane;
    if (dq32)
      *reinterpret_cast<float4*>(dq32 + off) = make_float4(x[0], x[1], x[2], x[3]);
    else
      *reinterpret_cast<uint2*>(dq + off) = make_uint2(pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]));
  }
}

}  // namespace

size_t fused_dq_acc_bytes(int64_t B, int64_t H, int64_t n_tiles) {
  return (size_t)B * (size_t)H * (size_t)n_tiles * 128 * kD * sizeof(float);
}

cudaError_t launch_sm100_bwd_fused(const Problem& pb, const Workspace& ws, const void* k,
                                   const void* v, const void* d_o, void* dq, void* dk, void* dv,
                                   cudaStream_t st, bool out_f32) {
  CUtensorMap tq, tk, tv, tdo, tdk, tdv;
  if (!make_qkv_map(&tq, ws.q_rot, pb.B, pb.S, pb.H, pb.D) ||
      !make_qkv_map(&tk, rope_on_load_bwd(pb) ? k : ws.k_rot, pb.B, pb.S, pb.H, pb.D) ||
      !make_qkv_map(&tv, v, pb.B, pb.S, pb.H, pb.D) ||
      !make_qkv_map(&tdo, d_o, pb.B, pb.S, pb.H, pb.D))
    return cudaErrorInvalidValue;
  const int64_t n_items = pb.B * pb.H * pb.n_tiles;
  if (n_items == 0) return cudaSuccess;
  FusedParams p{};
  p.seg = pb.seg;
  p.kseg = pb.kseg;
  p.tmin = ws.tile_min;
  p.tmax = ws.tile_max;
  p.ktmin = ws.ktile_min;
  p.ktmax = ws.ktile_max;
  p.k_hi = ws.k_hi;
  p.lse2 = ws.lse2_pad;
  p.dpad = ws.delta_pad;
  p.dq_acc = ws.dq_acc;
  p.dk = out_f32 ? nullptr : static_cast<__nv_bfloat16*>(dk);
  p.dv = out_f32 ? nullptr : static_cast<__nv_bfloat16*>(dv);
  p.dk32 = out_f32 ? static_cast<float*>(dk) : nullptr;
  p.dv32 = out_f32 ? static_cast<float*>(dv) : nullptr;
  p.status = ws.status;
  p.S = pb.S;
  p.H = (int)pb.H;
  p.B = (int)pb.B;
  p.n_tiles = (int)pb.n_tiles;
  p.scale = pb.scale;
  p.scale_log2 = pb.scale * 1.4426950408889634f;
  p.causal = pb.causal;
  p.rotate = pb.theta > 0.0;
  // a row piece starts at a multiple of 64 bytes from the base (32 bf16 or
  // fp32 columns), so 32-byte aligned bases make every 256-bit store aligned
  p.out_v8 = ((reinterpret_cast<uintptr_t>(dk) | reinterpret_cast<uintptr_t>(dv)) & 31u) == 0;
  // bf16 outputs leave by tensor stores where both maps encode (16-byte
  // aligned bases), else by the direct row stores
  memset(&tdk, 0, sizeof(tdk));
  memset(&tdv, 0, sizeof(tdv));
  p.tma_out = !out_f32 && make_bf16_store_map(&tdk, dk, pb.B, pb.S, pb.H, pb.D) &&
              make_bf16_store_map(&tdv, dv, pb.B, pb.S, pb.H, pb.D);
  p.rot_k = rope_on_load_bwd(pb);
  p.log2_theta = p.rotate ? log2(pb.theta) : 0.0;
  static std::once_flag attr_once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(attr_once, [] {
    attr_err = cudaFuncSetAttribute(attn_bwd_fused_kernel,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
  });
  if (attr_err != cudaSuccess) return attr_err;
  const int grid = (int)(n_items < sm_count() ? n_items : sm_count());
  attn_bwd_fused_kernel<<<grid, kThreads, kSmemBytes, st>>>(tq, tk, tv, tdo, tdk, tdv, p);
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_dq_finish(const Problem& pb, const Workspace& ws, void* dq, cudaStream_t st,
                             bool out_f32) {
  const int64_t blocks = 2 * pb.B * pb.H * pb.n_tiles;  // two half tiles each
  if (blocks == 0) return cudaSuccess;
  const int rotate = pb.theta > 0.0;
  constexpr int kFinSmem = kFinRows * kFinRow * (int)sizeof(float);
  static std::once_flag attr_once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(attr_once, [] {
    attr_err = cudaFuncSetAttribute(dq_finish_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    kFinSmem);
  });
  if (attr_err != cudaSuccess) return attr_err;
  dq_finish_kernel<<<(unsigned)blocks, kFinThreads, kFinSmem, st>>>(
      ws.dq_acc, out_f32 ? nullptr : static_cast<__nv_bfloat16*>(dq),
      out_f32 ? static_cast<float*>(dq) : nullptr, pb.S, (int)pb.H, (int)pb.n_tiles, pb.scale,
      rotate, rotate ? log2(pb.theta) : 0.0);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace lwm
