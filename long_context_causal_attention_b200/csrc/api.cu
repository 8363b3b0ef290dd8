// C ABI of liblwm_attn: argument checks, workspace layout and dispatch.
// The operations are defined in include/lwm_attn.h.
#include <atomic>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace lwm {

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

namespace {
std::atomic<uint64_t> g_launches{0};
std::mutex g_events_mu;
cudaEvent_t g_events[5] = {nullptr, nullptr, nullptr, nullptr, nullptr};

void record_event(int which, cudaStream_t st) {
  std::lock_guard<std::mutex> lk(g_events_mu);
  if (g_events[which]) cudaEventRecord(g_events[which], st);
}
}  // namespace

void note_launches(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

bool tensor_core_shape(const Problem& p) {
  return p.dtype == LWM_DTYPE_BF16 && p.D == 128 && p.S < ((int64_t)1 << 31);
}

// LWM_ATTN_FORCE_SIMT=1 routes every call to the CUDA-core kernels (used to
// cross-check the two kernel families against each other).
static bool force_simt() {
  static const bool v = [] {
    const char* e = std::getenv("LWM_ATTN_FORCE_SIMT");
    return e && e[0] == '1';
  }();
  return v;
}

// LWM_ATTN_FP32_SIMT=1 keeps fp32 problems on the CUDA-core kernels (full
// fp32 arithmetic) instead of the split-precision tensor-core path.
static bool fp32_simt() {
  static const bool v = [] {
    const char* e = std::getenv("LWM_ATTN_FP32_SIMT");
    return e && e[0] == '1';
  }();
  return v;
}

// fp32, head_dim 64 or 128: the shapes the split-precision kernels take.
bool x3_shape(const Problem& p) {
  return p.dtype == LWM_DTYPE_FP32 && (p.D == 64 || p.D == 128) && p.S < ((int64_t)1 << 31);
}

Path choose_fwd_path(const Problem& p) {
  if (force_simt() || !sm100_available()) return Path::kSimt;
  if (tensor_core_shape(p)) return Path::kSm100;
  if (x3_shape(p) && !fp32_simt()) return Path::kSm100X3;
  return Path::kSimt;
}

// LWM_ATTN_SPLIT_BWD=1 runs the tensor-core backward as two kernels (key-
// stationary dK/dV, query-stationary dQ) instead of the one-pass kernel.
static bool split_bwd() {
  static const bool v = [] {
    const char* e = std::getenv("LWM_ATTN_SPLIT_BWD");
    return e && e[0] == '1';
  }();
  return v;
}

Path choose_bwd_path(const Problem& p) {
  if (force_simt() || !sm100_available()) return Path::kSimt;
  if (tensor_core_shape(p)) return Path::kSm100;
  if (x3_shape(p) && !fp32_simt()) return Path::kSm100X3;
  return Path::kSimt;
}

size_t layout_workspace(const Problem& p, bool bwd, void* base, Workspace* ws) {
  char* b = static_cast<char*>(base);
  size_t off = 0;
  auto take = [&](size_t bytes) -> void* {
    off = align_up(off, 1024);
    void* r = b ? b + off : nullptr;
    off += bytes;
    return r;
  };
  Workspace w{};
  w.status = static_cast<DeviceStatus*>(take(sizeof(DeviceStatus)));
  const size_t tiles = (size_t)p.B * (size_t)p.n_tiles * sizeof(int32_t);
  w.tile_min = static_cast<int32_t*>(take(tiles));
  w.tile_max = static_cast<int32_t*>(take(tiles));
  w.ktile_min = static_cast<int32_t*>(take(tiles));
  w.ktile_max = static_cast<int32_t*>(take(tiles));
  if (p.kseg == p.seg) {
    w.ktile_min = w.tile_min;
    w.ktile_max = w.tile_max;
  }
  w.q_lo = static_cast<int32_t*>(take(tiles));
  w.k_hi = static_cast<int32_t*>(take(tiles));
  const size_t nel = (size_t)p.B * p.S * p.H * p.D;
  const bool x3 = bwd ? choose_bwd_path(p) == Path::kSm100X3 : choose_fwd_path(p) == Path::kSm100X3;
  if (x3) {
    // split planes replace the rotated copies (the split pre-pass rotates)
    w.qx_hi = take(nel * 2);
    w.qx_lo = take(nel * 2);
    w.kx_hi = take(nel * 2);
    w.kx_lo = take(nel * 2);
    w.vx_hi = take(nel * 2);
    w.vx_lo = take(nel * 2);
    if (bwd) {
      w.dox_hi = take(nel * 2);
      w.dox_lo = take(nel * 2);
      const size_t padded = (size_t)p.B * p.H * (size_t)p.n_tiles * kTile * sizeof(float);
      w.lse2_pad = static_cast<float*>(take(padded));
      w.delta_pad = static_cast<float*>(take(padded));
    }
  } else if (p.theta > 0.0) {
    // rotated copies the chosen kernels read: the tensor-core forward rotates
    // its Q tiles itself and the one-pass backward its K tiles
    const Path path = bwd ? choose_bwd_path(p) : choose_fwd_path(p);
    const bool on_load = path == Path::kSm100 &&
                         (bwd ? !split_bwd() && rope_on_load_bwd(p) : rope_on_load_fwd(p));
    if (!(on_load && !bwd)) w.q_rot = take(nel * p.elt);
    if (!(on_load && bwd)) w.k_rot = take(nel * p.elt);
  }
  if (bwd && !x3) {
    w.delta = static_cast<float*>(take((size_t)p.B * p.H * p.S * sizeof(float)));
    if (tensor_core_shape(p)) {
      const size_t padded = (size_t)p.B * p.H * (size_t)p.n_tiles * kTile * sizeof(float);
      w.lse2_pad = static_cast<float*>(take(padded));
      w.delta_pad = static_cast<float*>(take(padded));
      w.dq_acc = static_cast<float*>(take(fused_dq_acc_bytes(p.B, p.H, p.n_tiles)));
    }
  }
  w.bytes = align_up(off, 1024);
  if (ws) *ws = w;
  return w.bytes;
}

size_t layout_decode_workspace(const Problem& p, int64_t n_new, void* base, Workspace* ws) {
  char* b = static_cast<char*>(base);
  size_t off = 0;
  auto take = [&](size_t bytes) -> void* {
    off = align_up(off, 1024);
    void* r = b ? b + off : nullptr;
    off += bytes;
    return r;
  };
  Workspace w{};
  w.status = static_cast<DeviceStatus*>(take(sizeof(DeviceStatus)));
  const size_t tiles = (size_t)p.B * (size_t)p.n_tiles * sizeof(int32_t);
  w.tile_min = static_cast<int32_t*>(take(tiles));
  w.tile_max = static_cast<int32_t*>(take(tiles));
  w.ktile_min = w.tile_min;
  w.ktile_max = w.tile_max;
  const size_t parts = (size_t)p.B * p.H * (size_t)n_new *
                       (size_t)((p.S + kDecodeChunk - 1) / kDecodeChunk);
  w.dec_ml = static_cast<float*>(take(parts * 2 * sizeof(float)));
  w.dec_o = static_cast<float*>(take(parts * (size_t)p.D * sizeof(float)));
  w.bytes = align_up(off, 1024);
  if (ws) *ws = w;
  return w.bytes;
}

namespace {

bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

lwm_status make_problem(const lwm_attn_desc* d, Problem* p) {
  if (!d) return LWM_ERR_INVALID_ARG;
  if (d->batch < 0 || d->seqlen < 0 || d->heads < 1 || d->head_dim < 1) return LWM_ERR_INVALID_ARG;
  if (d->dtype != LWM_DTYPE_BF16 && d->dtype != LWM_DTYPE_FP32) return LWM_ERR_INVALID_ARG;
  if (d->causal != 0 && d->causal != 1) return LWM_ERR_INVALID_ARG;
  if (!std::isfinite(d->rope_theta) || !std::isfinite(d->softmax_scale)) return LWM_ERR_INVALID_ARG;
  if (d->head_dim != 64 && d->head_dim != 128) return LWM_ERR_UNSUPPORTED;
  if (d->heads > 65535 || d->batch > 65535) return LWM_ERR_UNSUPPORTED;
  if (d->seqlen > ((int64_t)1 << 33)) return LWM_ERR_UNSUPPORTED;
  if (reinterpret_cast<uintptr_t>(d->segment_ids) & 3u) return LWM_ERR_ALIGNMENT;
  p->B = d->batch;
  p->S = d->seqlen;
  p->H = d->heads;
  p->D = d->head_dim;
  p->dtype = d->dtype;
  p->causal = d->causal;
  p->theta = d->rope_theta;
  p->scale = d->softmax_scale > 0.f ? d->softmax_scale : (float)(1.0 / std::sqrt((double)d->head_dim));
  p->seg = d->segment_ids;
  p->kseg = d->segment_ids;
  p->n_tiles = (d->seqlen + kTile - 1) / kTile;
  p->elt = d->dtype == LWM_DTYPE_BF16 ? 2 : 4;
  return LWM_OK;
}

lwm_status check_ws(const Problem& p, bool bwd, void* ws, size_t ws_bytes, Workspace* w) {
  const size_t need = layout_workspace(p, bwd, nullptr, nullptr);
  if (!ws || ws_bytes < need) return LWM_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(ws) & 255u) return LWM_ERR_ALIGNMENT;
  layout_workspace(p, bwd, ws, w);
  return LWM_OK;
}

lwm_status cuda_status(cudaError_t e) { return e == cudaSuccess ? LWM_OK : LWM_ERR_CUDA; }

// Shared front half of forward and backward: status word, segment bounds,
// rotated q and k (those the workspace has room for: the kernels that rotate
// a tile themselves read the un-rotated input).
cudaError_t prologue(const Problem& p, Workspace& w, const void* q, const void* k, cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(w.status, 0, sizeof(DeviceStatus), st);
  if (e != cudaSuccess) return e;
  e = launch_segment_bounds(p, w, st);
  if (e != cudaSuccess) return e;
  if (p.theta > 0.0) {
    if (w.q_rot) e = launch_rope(p.B, p.S, p.H, p.D, p.dtype, p.theta, q, w.q_rot, 0, st);
    if (e == cudaSuccess && w.k_rot)
      e = launch_rope(p.B, p.S, p.H, p.D, p.dtype, p.theta, k, w.k_rot, 0, st);
  } else {
    w.q_rot = const_cast<void*>(q);
    w.k_rot = const_cast<void*>(k);
  }
  return e;
}

}  // namespace
}  // namespace lwm

namespace lwm {
namespace {
// Key segment ids of a block pair: both id arrays or neither.
lwm_status set_key_segments(Problem* p, const int32_t* k_segment_ids) {
  if ((p->seg == nullptr) != (k_segment_ids == nullptr)) return LWM_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(k_segment_ids) & 3u) return LWM_ERR_ALIGNMENT;
  p->kseg = k_segment_ids;
  return LWM_OK;
}

// out_f32: the outputs are fp32 whatever the input dtype (block partials of
// a ring); supported on the fp32 paths and the tensor-core bf16 path.
lwm_status attn_fwd(const lwm_attn_desc* desc, const int32_t* const* k_segment_ids,
                    const void* q, const void* k, const void* v, void* o, float* lse, void* ws,
                    size_t ws_bytes, void* stream, bool out_f32 = false) {
  Problem p{};
  lwm_status s = make_problem(desc, &p);
  if (s != LWM_OK) return s;
  if (k_segment_ids && (s = set_key_segments(&p, *k_segment_ids)) != LWM_OK) return s;
  if (p.B * p.S == 0) return LWM_OK;
  if (!q || !k || !v || !o || !lse) return LWM_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return LWM_ERR_ALIGNMENT;
  Workspace w{};
  s = check_ws(p, false, ws, ws_bytes, &w);
  if (s != LWM_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Path path = choose_fwd_path(p);
  const bool f32_out = out_f32 && p.dtype == LWM_DTYPE_BF16;
  if (f32_out && path != Path::kSm100) return LWM_ERR_UNSUPPORTED;
  cudaError_t e;
  if (path == Path::kSm100X3) {
    e = cudaMemsetAsync(w.status, 0, sizeof(DeviceStatus), st);
    if (e == cudaSuccess) e = launch_segment_bounds(p, w, st);
    if (e == cudaSuccess)
      e = launch_split(p.B, p.S, p.H, p.D, p.theta, static_cast<const float*>(q), w.qx_hi,
                       w.qx_lo, st);
    if (e == cudaSuccess)
      e = launch_split(p.B, p.S, p.H, p.D, p.theta, static_cast<const float*>(k), w.kx_hi, w.kx_lo, st);
    if (e == cudaSuccess)
      e = launch_split(p.B, p.S, p.H, p.D, 0.0, static_cast<const float*>(v), w.vx_hi, w.vx_lo, st);
    if (e != cudaSuccess) return LWM_ERR_CUDA;
    record_event(0, st);
    e = launch_sm100_fwd_x3(p, w, static_cast<float*>(o), lse, st);
    record_event(1, st);
    return cuda_status(e);
  }
  e = prologue(p, w, q, k, st);
  if (e != cudaSuccess) return LWM_ERR_CUDA;
  record_event(0, st);
  if (path == Path::kSm100)
    e = launch_sm100_fwd(p, w, q, v, o, lse, st, f32_out);
  else
    e = launch_simt_fwd(p, w, v, o, lse, st);
  record_event(1, st);
  return cuda_status(e);
}

lwm_status attn_bwd(const lwm_attn_desc* desc, const int32_t* const* k_segment_ids,
                    const void* q, const void* k, const void* v, const void* o, const float* lse,
                    const void* d_o, void* dq, void* dk, void* dv, void* ws, size_t ws_bytes,
                    void* stream, bool out_f32 = false) {
  Problem p{};
  lwm_status s = make_problem(desc, &p);
  if (s != LWM_OK) return s;
  if (k_segment_ids && (s = set_key_segments(&p, *k_segment_ids)) != LWM_OK) return s;
  if (p.B * p.S == 0) return LWM_OK;
  if (!q || !k || !v || !o || !lse || !d_o || !dq || !dk || !dv) return LWM_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) ||
      !aligned16(d_o) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return LWM_ERR_ALIGNMENT;
  Workspace w{};
  s = check_ws(p, true, ws, ws_bytes, &w);
  if (s != LWM_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Path path = choose_bwd_path(p);
  const bool f32_out = out_f32 && p.dtype == LWM_DTYPE_BF16;
  if (f32_out && (path != Path::kSm100 || split_bwd())) return LWM_ERR_UNSUPPORTED;
  cudaError_t e;
  if (path == Path::kSm100X3) {
    e = cudaMemsetAsync(w.status, 0, sizeof(DeviceStatus), st);
    if (e == cudaSuccess) e = launch_segment_bounds(p, w, st);
    const float* fq = static_cast<const float*>(q);
    const float* fk = static_cast<const float*>(k);
    if (e == cudaSuccess) e = launch_split(p.B, p.S, p.H, p.D, p.theta, fq, w.qx_hi, w.qx_lo, st);
    if (e == cudaSuccess) e = launch_split(p.B, p.S, p.H, p.D, p.theta, fk, w.kx_hi, w.kx_lo, st);
    if (e == cudaSuccess)
      e = launch_split(p.B, p.S, p.H, p.D, 0.0, static_cast<const float*>(v), w.vx_hi, w.vx_lo, st);
    if (e == cudaSuccess)
      e = launch_split(p.B, p.S, p.H, p.D, 0.0, static_cast<const float*>(d_o), w.dox_hi, w.dox_lo,
                       st);
    if (e == cudaSuccess) e = launch_bwd_prep(p, o, d_o, lse, w, st);
    if (e != cudaSuccess) return LWM_ERR_CUDA;
    record_event(2, st);
    e = launch_sm100_bwd_x3(p, w, dq, dk, dv, st);
    record_event(4, st);
    record_event(3, st);
    return cuda_status(e);
  }
  e = prologue(p, w, q, k, st);
  if (e != cudaSuccess) return LWM_ERR_CUDA;
  if (path == Path::kSm100) {
    e = launch_bwd_prep(p, o, d_o, lse, w, st);
    if (e == cudaSuccess && !split_bwd())
      e = cudaMemsetAsync(w.dq_acc, 0, fused_dq_acc_bytes(p.B, p.H, p.n_tiles), st);
    if (e != cudaSuccess) return LWM_ERR_CUDA;
    record_event(2, st);
    if (split_bwd()) {
      e = launch_sm100_bwd_dkdv(p, w, v, d_o, dk, dv, st);
      record_event(4, st);
      if (e == cudaSuccess) e = launch_sm100_bwd_dq(p, w, v, d_o, dq, st);
    } else {
      e = launch_sm100_bwd_fused(p, w, k, v, d_o, dq, dk, dv, st, f32_out);
      record_event(4, st);
      if (e == cudaSuccess) e = launch_dq_finish(p, w, dq, st, f32_out);
    }
    record_event(3, st);
    return cuda_status(e);
  }
  e = launch_delta(p, o, d_o, w.delta, st);
  if (e != cudaSuccess) return LWM_ERR_CUDA;
  record_event(2, st);
  e = launch_simt_bwd_dkdv(p, w, v, lse, d_o, dk, dv, st);
  record_event(4, st);
  if (e == cudaSuccess) e = launch_simt_bwd_dq(p, w, v, lse, d_o, dq, st);
  record_event(3, st);
  return cuda_status(e);
}

}  // namespace
}  // namespace lwm

using namespace lwm;

extern "C" {

size_t lwm_attn_workspace_size(const lwm_attn_desc* desc, int is_bwd) {
  Problem p{};
  if (make_problem(desc, &p) != LWM_OK) return 0;
  return layout_workspace(p, is_bwd != 0, nullptr, nullptr);
}


lwm_status lwm_attn_fwd(const lwm_attn_desc* desc, const void* q, const void* k, const void* v,
                        void* o, float* lse, void* ws, size_t ws_bytes, void* stream) {
  return attn_fwd(desc, nullptr, q, k, v, o, lse, ws, ws_bytes, stream);
}

lwm_status lwm_attn_bwd(const lwm_attn_desc* desc, const void* q, const void* k, const void* v,
                        const void* o, const float* lse, const void* d_o, void* dq, void* dk,
                        void* dv, void* ws, size_t ws_bytes, void* stream) {
  return attn_bwd(desc, nullptr, q, k, v, o, lse, d_o, dq, dk, dv, ws, ws_bytes, stream);
}

lwm_status lwm_attn_fwd_pair(const lwm_attn_desc* desc, const int32_t* k_segment_ids,
                             const void* q, const void* k, const void* v, void* o, float* lse,
                             void* ws, size_t ws_bytes, void* stream) {
  return attn_fwd(desc, &k_segment_ids, q, k, v, o, lse, ws, ws_bytes, stream);
}

lwm_status lwm_attn_bwd_pair(const lwm_attn_desc* desc, const int32_t* k_segment_ids,
                             const void* q, const void* k, const void* v, const void* o,
                             const float* lse, const void* d_o, void* dq, void* dk, void* dv,
                             void* ws, size_t ws_bytes, void* stream) {
  return attn_bwd(desc, &k_segment_ids, q, k, v, o, lse, d_o, dq, dk, dv, ws, ws_bytes, stream);
}

lwm_status lwm_attn_fwd_pair_f32(const lwm_attn_desc* desc, const int32_t* k_segment_ids,
                                 const void* q, const void* k, const void* v, float* o, float* lse,
                                 void* ws, size_t ws_bytes, void* stream) {
  return attn_fwd(desc, &k_segment_ids, q, k, v, o, lse, ws, ws_bytes, stream, true);
}

lwm_status lwm_attn_bwd_pair_f32(const lwm_attn_desc* desc, const int32_t* k_segment_ids,
                                 const void* q, const void* k, const void* v, const void* o,
                                 const float* lse, const void* d_o, float* dq, float* dk, float* dv,
                                 void* ws, size_t ws_bytes, void* stream) {
  return attn_bwd(desc, &k_segment_ids, q, k, v, o, lse, d_o, dq, dk, dv, ws, ws_bytes, stream,
                  true);
}

size_t lwm_attn_decode_workspace_size(const lwm_attn_desc* desc, int64_t n_new) {
  Problem p{};
  if (make_problem(desc, &p) != LWM_OK || n_new < 1 || n_new > p.S) return 0;
  return layout_decode_workspace(p, n_new, nullptr, nullptr);
}

lwm_status lwm_attn_decode(const lwm_attn_desc* desc, int64_t n_new, const void* q,
                           const void* k_cache, const void* v_cache, void* o, float* lse,
                           void* ws, size_t ws_bytes, void* stream) {
  Problem p{};
  lwm_status s = make_problem(desc, &p);
  if (s != LWM_OK) return s;
  if (p.dtype != LWM_DTYPE_BF16 || p.D != 128) return LWM_ERR_UNSUPPORTED;
  if (n_new < 1 || n_new > p.S) return p.B == 0 && n_new >= 0 ? LWM_OK : LWM_ERR_INVALID_ARG;
  if (n_new > LWM_DECODE_MAX_NEW) return LWM_ERR_UNSUPPORTED;
  if (p.B == 0) return LWM_OK;
  if ((p.S + kDecodeChunk - 1) / kDecodeChunk > INT32_MAX) return LWM_ERR_UNSUPPORTED;
  if (!q || !k_cache || !v_cache || !o || !lse) return LWM_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o) ||
      !aligned16(lse))
    return LWM_ERR_ALIGNMENT;
  const size_t need = layout_decode_workspace(p, n_new, nullptr, nullptr);
  if (!ws || ws_bytes < need) return LWM_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(ws) & 255u) return LWM_ERR_ALIGNMENT;
  Workspace w{};
  layout_decode_workspace(p, n_new, ws, &w);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(w.status, 0, sizeof(DeviceStatus), st);
  if (e == cudaSuccess) e = launch_segment_bounds(p, w, st, false);
  if (e != cudaSuccess) return LWM_ERR_CUDA;
  record_event(0, st);
  e = launch_decode(p, w, n_new, q, k_cache, v_cache, o, lse, st);
  record_event(1, st);
  return cuda_status(e);
}

lwm_status lwm_rope_apply(int64_t batch, int64_t seqlen, int64_t heads, int64_t head_dim,
                          int32_t dtype, double theta, const void* x, void* y, int inverse,
                          void* stream) {
  if (batch < 0 || seqlen < 0 || heads < 1 || head_dim < 2 || (head_dim & 1)) return LWM_ERR_INVALID_ARG;
  if (dtype != LWM_DTYPE_BF16 && dtype != LWM_DTYPE_FP32) return LWM_ERR_INVALID_ARG;
  if (!std::isfinite(theta)) return LWM_ERR_INVALID_ARG;
  const int vec = dtype == LWM_DTYPE_BF16 ? 8 : 4;
  if (head_dim % vec != 0 || head_dim > 512) return LWM_ERR_UNSUPPORTED;
  if (batch * seqlen == 0) return LWM_OK;
  if (!x || !y) return LWM_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(y)) return LWM_ERR_ALIGNMENT;
  return cuda_status(launch_rope(batch, seqlen, heads, head_dim, dtype, theta, x, y, inverse,
                                 static_cast<cudaStream_t>(stream)));
}

lwm_status lwm_rope_apply_at(int64_t batch, int64_t seqlen, int64_t heads, int64_t head_dim,
                             int32_t dtype, double theta, int64_t position_offset, const void* x,
                             void* y, int inverse, void* stream) {
  if (batch < 0 || seqlen < 0 || heads < 1 || head_dim < 2 || (head_dim & 1)) return LWM_ERR_INVALID_ARG;
  if (dtype != LWM_DTYPE_BF16 && dtype != LWM_DTYPE_FP32) return LWM_ERR_INVALID_ARG;
  if (!std::isfinite(theta) || position_offset < 0) return LWM_ERR_INVALID_ARG;
  const int vec = dtype == LWM_DTYPE_BF16 ? 8 : 4;
  if (head_dim % vec != 0 || head_dim > 512) return LWM_ERR_UNSUPPORTED;
  if (batch * seqlen == 0) return LWM_OK;
  if (!x || !y) return LWM_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(y)) return LWM_ERR_ALIGNMENT;
  return cuda_status(launch_rope(batch, seqlen, heads, head_dim, dtype, theta, x, y, inverse,
                                 static_cast<cudaStream_t>(stream), position_offset));
}

lwm_status lwm_attn_merge(int64_t batch, int64_t seqlen, int64_t heads, int64_t head_dim,
                          int32_t dtype, float* o_acc, float* lse_acc, const void* o_part,
                          const float* lse_part, void* stream) {
  if (batch < 0 || seqlen < 0 || heads < 1 || head_dim < 1) return LWM_ERR_INVALID_ARG;
  if (dtype != LWM_DTYPE_BF16 && dtype != LWM_DTYPE_FP32) return LWM_ERR_INVALID_ARG;
  if (batch * seqlen == 0) return LWM_OK;
  if (!o_acc || !lse_acc || !o_part || !lse_part) return LWM_ERR_INVALID_ARG;
  return cuda_status(launch_attn_merge(batch, seqlen, heads, head_dim, dtype, o_acc, lse_acc,
                                       o_part, lse_part, static_cast<cudaStream_t>(stream)));
}

lwm_status lwm_accumulate(int64_t n, int32_t dtype, float* acc, const void* x, void* stream) {
  if (n < 0 || (dtype != LWM_DTYPE_BF16 && dtype != LWM_DTYPE_FP32)) return LWM_ERR_INVALID_ARG;
  if (n == 0) return LWM_OK;
  if (!acc || !x) return LWM_ERR_INVALID_ARG;
  return cuda_status(launch_accumulate(n, dtype, acc, x, static_cast<cudaStream_t>(stream)));
}

lwm_status lwm_convert_f32(int64_t n, int32_t dtype, const float* x, void* y, void* stream) {
  if (n < 0 || (dtype != LWM_DTYPE_BF16 && dtype != LWM_DTYPE_FP32)) return LWM_ERR_INVALID_ARG;
  if (n == 0) return LWM_OK;
  if (!x || !y) return LWM_ERR_INVALID_ARG;
  return cuda_status(launch_convert_f32(n, dtype, x, y, static_cast<cudaStream_t>(stream)));
}

size_t lwm_packed_ce_workspace_size(int64_t batch, int64_t seqlen) {
  if (batch < 0 || seqlen < 0) return 0;
  return packed_ce_workspace_bytes(batch, seqlen);
}

lwm_status lwm_packed_cross_entropy(int64_t batch, int64_t seqlen, int64_t vocab, int32_t dtype,
                                    const void* logits, const int32_t* targets,
                                    const int32_t* segment_ids, float* loss, void* dlogits,
                                    void* ws, size_t ws_bytes, void* stream) {
  if (batch < 0 || seqlen < 0 || vocab < 1) return LWM_ERR_INVALID_ARG;
  if (dtype != LWM_DTYPE_BF16 && dtype != LWM_DTYPE_FP32) return LWM_ERR_INVALID_ARG;
  if (batch > 2147483647 || batch * seqlen > 2147483647) return LWM_ERR_UNSUPPORTED;
  if (vocab > packed_ce_max_vocab(dtype)) return LWM_ERR_UNSUPPORTED;
  if (vocab % (dtype == LWM_DTYPE_BF16 ? 8 : 4) != 0) return LWM_ERR_UNSUPPORTED;  // 16-byte rows
  if (!loss) return LWM_ERR_INVALID_ARG;
  if (batch * seqlen == 0) {
    return cuda_status(cudaMemsetAsync(loss, 0, sizeof(float), static_cast<cudaStream_t>(stream)));
  }
  if (!logits || !targets) return LWM_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(targets) & 3u) || (reinterpret_cast<uintptr_t>(segment_ids) & 3u) ||
      (reinterpret_cast<uintptr_t>(logits) & 15u) || (reinterpret_cast<uintptr_t>(dlogits) & 15u))
    return LWM_ERR_ALIGNMENT;
  if (!ws || ws_bytes < packed_ce_workspace_bytes(batch, seqlen)) return LWM_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(ws) & 255u) return LWM_ERR_ALIGNMENT;
  return cuda_status(launch_packed_ce(batch, seqlen, vocab, dtype, logits, targets, segment_ids,
                                      loss, dlogits, ws, static_cast<cudaStream_t>(stream)));
}

lwm_status lwm_attn_selftest_wait(void* ws, size_t ws_bytes, int64_t limit_cycles, int arrive,
                                  void* stream) {
  if (!ws || ws_bytes < sizeof(DeviceStatus) || limit_cycles < 0) return LWM_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(ws) & 255u) return LWM_ERR_ALIGNMENT;
  return cuda_status(launch_selftest_wait(static_cast<DeviceStatus*>(ws), (long long)limit_cycles,
                                          arrive != 0, static_cast<cudaStream_t>(stream)));
}

lwm_status lwm_attn_read_status(const void* ws, void* stream) {
  if (!ws) return LWM_ERR_INVALID_ARG;
  int32_t code = 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(&code, ws, sizeof(code), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return LWM_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return LWM_ERR_CUDA;
  return code == 0 ? LWM_OK : static_cast<lwm_status>(code);
}

const char* lwm_status_string(lwm_status status) {
  switch (status) {
    case LWM_OK: return "LWM_OK";
    case LWM_ERR_INVALID_ARG: return "LWM_ERR_INVALID_ARG: invalid argument";
    case LWM_ERR_UNSUPPORTED: return "LWM_ERR_UNSUPPORTED: unsupported configuration";
    case LWM_ERR_ALIGNMENT: return "LWM_ERR_ALIGNMENT: pointer not 16-byte aligned (workspace: 256)";
    case LWM_ERR_WORKSPACE: return "LWM_ERR_WORKSPACE: workspace missing or too small";
    case LWM_ERR_CUDA: return "LWM_ERR_CUDA: CUDA runtime error";
    case LWM_ERR_TIMEOUT: return "LWM_ERR_TIMEOUT: a bounded device wait ran out";
  }
  return "unknown lwm_status";
}

void lwm_attn_set_timing_events(void* fwd_start, void* fwd_stop, void* bwd_start,
                                void* bwd_stop, void* bwd_split) {
  std::lock_guard<std::mutex> lk(g_events_mu);
  g_events[0] = static_cast<cudaEvent_t>(fwd_start);
  g_events[1] = static_cast<cudaEvent_t>(fwd_stop);
  g_events[2] = static_cast<cudaEvent_t>(bwd_start);
  g_events[3] = static_cast<cudaEvent_t>(bwd_stop);
  g_events[4] = static_cast<cudaEvent_t>(bwd_split);
}

uint64_t lwm_attn_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

}  // extern "C"
