// Host-side internals shared by the translation units of liblwm_attn.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "lwm_attn.h"

namespace lwm {

struct DeviceStatus;

// Validated problem, in the form the launchers take.
struct Problem {
  int64_t B, S, H, D;
  int dtype;          // lwm_dtype
  int causal;
  double theta;       // <= 0: no rotation
  float scale;        // resolved softmax scale (> 0)
  const int32_t* seg; // may be null; segment ids of the queries
  const int32_t* kseg; // segment ids of the keys: seg itself, except for a block pair
  int64_t n_tiles;    // ceil(S / 128)
  size_t elt;         // bytes per element of dtype
};

// Carved-up workspace.  Every region is 1024-byte aligned.
struct Workspace {
  DeviceStatus* status;
  int32_t* tile_min;   // [B, n_tiles] smallest non-negative id in the tile (INT32_MAX if none)
  int32_t* tile_max;   // [B, n_tiles] largest id in the tile (-1 if none)
  int32_t* ktile_min;  // the same bounds for the key ids (alias of tile_min/max
  int32_t* ktile_max;  //   unless the keys carry their own ids)
  int32_t* q_lo;       // [B, n_tiles] first key tile a query tile may need
  int32_t* k_hi;       // [B, n_tiles] last query tile a key tile may feed
  void* q_rot;         // [B, S, H, D] rotated q (dtype)
  void* k_rot;         // [B, S, H, D] rotated k (dtype)
  float* delta;        // [B, H, S] fp32 dot(dO, O) per row (backward, CUDA-core path)
  float* lse2_pad;     // [B, H, n_tiles*128] LSE*log2(e) or +inf (backward, tensor-core path)
  float* delta_pad;    // [B, H, n_tiles*128] dot(dO, O) or 0 (backward, tensor-core path)
  float* dq_acc;       // [B*H, n_tiles, 32, 128, 4] fp32 dQ~ sums (backward, tensor-core path)
  // fp32 on the tensor cores: bf16 hi / lo planes [B, S, H, D] of the rotated
  // q and k and of v (forward)
  void* qx_hi;
  void* qx_lo;
  void* kx_hi;
  void* kx_lo;
  void* vx_hi;
  void* vx_lo;
  void* dox_hi;        // and of dO (backward)
  void* dox_lo;
  float* dec_ml;       // [B, H, T, n_chunks, 2] decode chunk max and sum (log2 domain)
  float* dec_o;        // [B, H, T, n_chunks, D] decode chunk sums of p * v
  size_t bytes;        // total bytes the layout needs
};

// kSm100X3: fp32 data on the bf16 tensor cores through hi/lo splits.
enum class Path { kSimt = 0, kSm100 = 1, kSm100X3 = 2 };

// RoPE applied by the tensor-core kernels to their stationary tiles in
// shared memory instead of a rotated copy in the workspace, at every
// length: the one-pass backward rotates its K tiles, the forward its Q
// tiles.  Each tile is rotated once per work item, which costs less than
// the pre-pass it replaces, even on the short work items of packed rows.
inline bool rope_on_load_fwd(const Problem& p) { return p.theta > 0.0; }
inline bool rope_on_load_bwd(const Problem& p) { return p.theta > 0.0; }

// Which kernels serve the forward / backward of this problem on this device.
Path choose_fwd_path(const Problem& p);
Path choose_bwd_path(const Problem& p);
// bf16, head_dim 128: the shape the tensor-core kernels are built for.
bool tensor_core_shape(const Problem& p);
bool sm100_available();

// Instrumentation: kernels launched so far (process-wide).
void note_launches(int n);
size_t layout_workspace(const Problem& p, bool bwd, void* base, Workspace* ws);

// Launchers (return the first CUDA error, or cudaSuccess).
// pos0: position of token 0 of each row (p = pos0 + index in the row).
cudaError_t launch_rope(int64_t B, int64_t S, int64_t H, int64_t D, int dtype, double theta,
                        const void* x, void* y, int inverse, cudaStream_t st, int64_t pos0 = 0);
// fp32 x [B,S,H,D] -> bf16 planes hi = bf16(y), lo = bf16(y - hi) with y =
// R(p) x when theta > 0 (p = pos0 + index in the row), else y = x.
cudaError_t launch_split(int64_t B, int64_t S, int64_t H, int64_t D, double theta, const float* x,
                         void* hi, void* lo, cudaStream_t st, int64_t pos0 = 0);
// Block results of one sequence split into key blocks (ring order):
// o_acc/lse_acc <- exact log-sum-exp merge with (o_part, lse_part).
cudaError_t launch_attn_merge(int64_t B, int64_t S, int64_t H, int64_t D, int dtype, float* o_acc,
                              float* lse_acc, const void* o_part, const float* lse_part,
                              cudaStream_t st);
size_t packed_ce_workspace_bytes(int64_t B, int64_t S);
int64_t packed_ce_max_vocab(int dtype);
cudaError_t launch_packed_ce(int64_t B, int64_t S, int64_t V, int dtype, const void* logits,
                             const int32_t* targets, const int32_t* seg, float* loss,
                             void* dlogits, void* ws, cudaStream_t st);
cudaError_t launch_accumulate(int64_t n, int dtype, float* acc, const void* x, cudaStream_t st);
cudaError_t launch_convert_f32(int64_t n, int dtype, const float* x, void* y, cudaStream_t st);
// ranges = false computes only the per-tile bounds (no q_lo / k_hi).
cudaError_t launch_segment_bounds(const Problem& p, const Workspace& ws, cudaStream_t st,
                                  bool ranges = true);
// Keys per CTA of the decode kernel (one partial softmax per chunk).
constexpr int64_t kDecodeChunk = 512;
size_t layout_decode_workspace(const Problem& p, int64_t n_new, void* base, Workspace* ws);
cudaError_t launch_decode(const Problem& p, const Workspace& ws, int64_t n_new, const void* q,
                          const void* k_cache, const void* v_cache, void* o, float* lse,
                          cudaStream_t st);
cudaError_t launch_delta(const Problem& p, const void* o, const void* d_o, float* delta,
                         cudaStream_t st);

// q un-rotated (the kernel applies RoPE to its Q tiles), k rotated in ws.k_rot.
// o_f32: O written as fp32 (block partials a ring merges) instead of bf16.
cudaError_t launch_sm100_fwd(const Problem& p, const Workspace& ws, const void* q, const void* v,
                             void* o, float* lse, cudaStream_t st, bool o_f32 = false);
// fp32 backward on the tensor cores from the split planes in ws and the
// padded LSE*log2(e) and dot(dO, O) (head_dim 64 or 128); dq, dk, dv fp32.
cudaError_t launch_sm100_bwd_x3(const Problem& p, const Workspace& ws, void* dq, void* dk,
                                void* dv, cudaStream_t st);
// fp32 forward on the tensor cores from the split planes in ws (head_dim 64 or 128).
cudaError_t launch_sm100_fwd_x3(const Problem& p, const Workspace& ws, float* o, float* lse,
                                cudaStream_t st);

cudaError_t launch_bwd_prep(const Problem& p, const void* o, const void* d_o, const float* lse,
                            const Workspace& ws, cudaStream_t st);
cudaError_t launch_sm100_bwd_dkdv(const Problem& p, const Workspace& ws, const void* v,
                                  const void* d_o, void* dk, void* dv, cudaStream_t st);
cudaError_t launch_sm100_bwd_dq(const Problem& p, const Workspace& ws, const void* v,
                                const void* d_o, void* dq, cudaStream_t st);
// One-pass backward: dK, dV, and dQ~ partial sums added into ws.dq_acc
// (which must be zero beforehand); launch_dq_finish turns those into bf16 dq.
size_t fused_dq_acc_bytes(int64_t B, int64_t H, int64_t n_tiles);
// k un-rotated (the kernel applies RoPE to its K tiles), q rotated in ws.q_rot.
cudaError_t launch_sm100_bwd_fused(const Problem& p, const Workspace& ws, const void* k,
                                   const void* v, const void* d_o, void* dq, void* dk, void* dv,
                                   cudaStream_t st, bool out_f32 = false);
cudaError_t launch_dq_finish(const Problem& p, const Workspace& ws, void* dq, cudaStream_t st,
                             bool out_f32 = false);

// Bounded-wait self-test: one CTA waits on an mbarrier (armed by an arrival
// or not) for at most limit_cycles; a wait that runs out records
// LWM_ERR_TIMEOUT in *status.
cudaError_t launch_selftest_wait(DeviceStatus* status, long long limit_cycles, int arrive,
                                 cudaStream_t st);
cudaError_t launch_simt_fwd(const Problem& p, const Workspace& ws, const void* v, void* o,
                            float* lse, cudaStream_t st);
cudaError_t launch_simt_bwd_dkdv(const Problem& p, const Workspace& ws, const void* v,
                                 const float* lse, const void* d_o, void* dk, void* dv,
                                 cudaStream_t st);
cudaError_t launch_simt_bwd_dq(const Problem& p, const Workspace& ws, const void* v,
                               const float* lse, const void* d_o, void* dq, cudaStream_t st);

}  // namespace lwm
