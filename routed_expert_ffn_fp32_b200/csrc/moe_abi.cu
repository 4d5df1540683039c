// C-ABI entry points (include/moe.h): argument checks, workspace carving and
// the launch sequence of each call.  No entry point allocates device memory
// or synchronises the host, except moe_get_error().
#include <cstdint>
#include <cstring>
#include <mutex>

#include "moe_internal.cuh"

namespace moe {

DeviceInfo device_info() {
  static std::mutex mu;
  static DeviceInfo cache[64];
  static bool have[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lock(mu);
  if (dev < 0 || dev >= 64) dev = 0;
  if (!have[dev]) {
    DeviceInfo di{};
    cudaDeviceGetAttribute(&di.sm_count, cudaDevAttrMultiProcessorCount, dev);
    cudaDeviceGetAttribute(&di.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (di.sm_count <= 0) di.sm_count = 148;
    cache[dev] = di;
    have[dev] = true;
  }
  return cache[dev];
}

}  // namespace moe

using namespace moe;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

moe_status_t check_shape(const moe_shape_t& s) {
  if (s.T < 1 || s.T > 65536) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (s.H < 32 || s.H > 16384 || s.H % 32) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (s.I < 32 || s.I > 16384 || s.I % 32) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (s.E < 1 || s.E > kMaxExperts) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (s.k < 1 || s.k > kMaxTopK || s.k > s.E) return MOE_ERR_UNSUPPORTED_SHAPE;
  return MOE_OK;
}

// The expert-FFN entry: k only describes the pair layout (p = t*k + j), so it
// may exceed the number of experts passed (one rank's share of them).
moe_status_t check_ffn_shape(const moe_shape_t& s) {
  moe_shape_t r = s;
  r.k = 1;
  if (check_shape(r) != MOE_OK || s.k < 1 || s.k > kMaxTopK) return MOE_ERR_UNSUPPORTED_SHAPE;
  return MOE_OK;
}

moe_status_t check_ptrs(std::initializer_list<const void*> required) {
  for (const void* p : required)
    if (p == nullptr || !aligned16(p)) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

bool opt_ok(const void* p) { return p == nullptr || aligned16(p); }

moe_status_t check_experts(const moe_mxfp4_experts_t* ex, int n) {
  if (ex == nullptr || ex->n_experts != n) return MOE_ERR_INVALID_ARG;
  return check_ptrs({ex->gate_q, ex->gate_s, ex->up_q, ex->up_s, ex->down_q, ex->down_s});
}

ExpertPtrs ptrs_of(const moe_mxfp4_experts_t* ex) {
  ExpertPtrs p{};
  if (ex) {
    p.gq = ex->gate_q;
    p.gs = ex->gate_s;
    p.uq = ex->up_q;
    p.us = ex->up_s;
    p.dq = ex->down_q;
    p.ds = ex->down_s;
  }
  return p;
}

moe_status_t cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return MOE_OK;
  cudaGetLastError();  // clear a sticky launch-configuration error
  return MOE_ERR_CUDA;
}

bool valid_path(int32_t path) {
  return path == MOE_PATH_AUTO || path == MOE_PATH_GEMV || path == MOE_PATH_GEMM;
}
bool valid_precision(int32_t p) { return p == MOE_ACT_EXACT || p == MOE_ACT_MXFP4; }

// Batches from which AUTO takes the tensor-core path (MXFP4 activations only):
// below it the weight stream dominates and the CUDA-core GEMV is as fast.
// AUTO: the tensor-core kernels whenever the activations are MXFP4 (measured
// on the 8-layer batch sweep, they beat the CUDA-core kernels from one token
// up); exact activations always take the CUDA-core kernels.
int resolve_path(int32_t path, int32_t precision, const moe_shape_t& s) {
  if (path == MOE_PATH_GEMM)
    return (precision == MOE_ACT_MXFP4 && gemm_supported(s)) ? MOE_PATH_GEMM : -1;
  if (path == MOE_PATH_AUTO && precision == MOE_ACT_MXFP4 && gemm_supported(s))
    return MOE_PATH_GEMM;
  return MOE_PATH_GEMV;
}

GemmBuffers gemm_buffers(void* ws, const WsLayout& L, int E);

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<unsigned char*>(ws) + off);
}

// CUDA-core FFN: the row-block mma.sync GEMV where the shape fits it, else the
// K-split GEMV.  A single token takes the K-split GEMV: with one token per
// expert every row block of the row-block GEMV is split over many warps, and
// the whole layer measured faster on the K-split kernel (decode64 36.7 ->
// 33.1 us, finegrained 73.0 -> 69.9 us).
cudaError_t launch_gemv_path(const FfnArgs& a, void* ws, const WsLayout& L, cudaStream_t s) {
  const moe_shape_t shape{a.T, a.H, a.I, a.E, a.k};
  if (a.xh != nullptr && a.T >= 2 && lane_supported(shape)) {
    const cudaError_t e =
        launch_ffn_lane(a, at<float>(ws, L.lane_part), at<uint32_t>(ws, L.lane_cnt), s);
    if (e != cudaErrorNotSupported) return e;
  }
  return launch_ffn_gemv(a, s);
}


constexpr int kFusedRouteMaxT = 32;

GemmBuffers gemm_buffers(void* ws, const WsLayout& L, int E) {
  GemmBuffers g{};
  g.xq = at<uint8_t>(ws, L.xq);
  g.xs = at<uint8_t>(ws, L.xs);
  g.hq = at<uint8_t>(ws, L.hq);
  g.hs = at<uint8_t>(ws, L.hs);
  g.item_off0 = at<int32_t>(ws, L.item_off);
  g.item_off1 = g.item_off0 + (E + 2);
  return g;
}

}  // namespace

extern "C" {

size_t moe_workspace_bytes(moe_shape_t shape, int32_t path, int32_t precision,
                           int32_t has_shared) {
  if (check_ffn_shape(shape) != MOE_OK || !valid_path(path) || !valid_precision(precision)) return 0;
  const int gemm = path != MOE_PATH_GEMV;
  return ws_layout(shape, has_shared != 0, gemm).total;
}

moe_status_t moe_workspace_init(void* ws, size_t ws_bytes, void* stream) {
  if (ws == nullptr || !aligned16(ws) || ws_bytes < 128) return MOE_ERR_INVALID_ARG;
  return cuda_status(cudaMemsetAsync(ws, 0, ws_bytes, static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_workspace_set_limits(void* ws, uint32_t wait_us, uint32_t debug, void* stream) {
  if (ws == nullptr || !aligned16(ws)) return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_set_words(static_cast<uint32_t*>(ws) + 2, wait_us, debug,
                                      static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_route_topk(const uint16_t* x, const float* w_router, const float* bias,
                            moe_shape_t shape, float* logits_out, int32_t* topk_idx,
                            float* topk_w, void* ws, size_t ws_bytes, void* stream) {
  moe_status_t st = check_shape(shape);
  if (st != MOE_OK) return st;
  st = check_ptrs({x, w_router, topk_idx, topk_w, ws});
  if (st != MOE_OK) return st;
  if (!opt_ok(bias) || !opt_ok(logits_out)) return MOE_ERR_INVALID_ARG;
  const WsLayout L = ws_layout(shape, 0, 0);
  if (ws_bytes < L.h) return MOE_ERR_WORKSPACE;
  RouteArgs a{};
  a.x = x;
  a.w_router = w_router;
  a.bias = bias;
  a.logits = logits_out ? logits_out : at<float>(ws, L.logits);
  a.idx = topk_idx;
  a.w = topk_w;
  a.counter = at<uint32_t>(ws, L.counters);
  a.err = at<int>(ws, L.err);
  a.T = shape.T;
  a.H = shape.H;
  a.E = shape.E;
  a.k = shape.k;
  // the layout's regions past the routing ones hold the router's K-split sums
  a.lpart = at<float>(ws, L.h);
  a.lpart_bytes = (ws_bytes < L.total ? ws_bytes : L.total) - L.h;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_route_logits(a, false, s);
  if (e == cudaSuccess) e = launch_topk(a, s);
  return cuda_status(e);
}

moe_status_t moe_bucket(const int32_t* topk_idx, moe_shape_t shape, int32_t* counts,
                        int32_t* offsets, int32_t* entries, void* ws, size_t ws_bytes,
                        void* stream) {
  moe_status_t st = check_shape(shape);
  if (st != MOE_OK) return st;
  st = check_ptrs({topk_idx, counts, offsets, entries, ws});
  if (st != MOE_OK) return st;
  const WsLayout L = ws_layout(shape, 0, 0);
  if (ws_bytes < L.h) return MOE_ERR_WORKSPACE;
  RouteArgs a{};
  a.idx = const_cast<int32_t*>(topk_idx);
  a.counts = counts;
  a.offsets = offsets;
  a.entries = entries;
  a.plan = at<int32_t>(ws, L.plan);
  a.err = at<int>(ws, L.err);
  a.T = shape.T;
  a.H = shape.H;
  a.E = shape.E;
  a.k = shape.k;
  // per-chunk counts of the multi-CTA bucket, inside this shape's layout
  a.lpart = at<float>(ws, L.h);
  a.lpart_bytes = (ws_bytes < L.total ? ws_bytes : L.total) - L.h;
  return cuda_status(launch_bucket(a, static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_expert_ffn_mxfp4(const moe_mxfp4_experts_t* experts,
                                  const moe_mxfp4_experts_t* shared, const uint16_t* x,
                                  const int32_t* offsets, const int32_t* entries,
                                  moe_shape_t shape, int32_t path, int32_t precision,
                                  float* partial_out, void* ws, size_t ws_bytes, void* stream) {
  moe_status_t st = check_ffn_shape(shape);
  if (st != MOE_OK) return st;
  if (!valid_path(path) || !valid_precision(precision)) return MOE_ERR_INVALID_ARG;
  st = check_experts(experts, shape.E);
  if (st != MOE_OK) return st;
  if (shared && (st = check_experts(shared, 1)) != MOE_OK) return st;
  st = check_ptrs({x, offsets, entries, partial_out, ws});
  if (st != MOE_OK) return st;
  const int rp = resolve_path(path, precision, shape);
  if (rp < 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  const int has_shared = shared != nullptr;
  const WsLayout L = ws_layout(shape, has_shared, rp == MOE_PATH_GEMM);
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  RouteArgs r{};
  r.offsets = const_cast<int32_t*>(offsets);
  r.plan = at<int32_t>(ws, L.plan);
  r.err = at<int>(ws, L.err);
  r.T = shape.T;
  r.H = shape.H;
  r.E = shape.E;
  r.k = shape.k;
  cudaError_t e = launch_plan(r, s);
  if (e != cudaSuccess) return cuda_status(e);
  FfnArgs a{};
  a.ex = ptrs_of(experts);
  a.sh = ptrs_of(shared);
  a.x = x;
  a.offsets = offsets;
  a.entries = entries;
  a.plan = r.plan;
  a.h = at<float>(ws, L.h);
  a.partial = partial_out;
  a.err = r.err;
  a.T = shape.T;
  a.H = shape.H;
  a.I = shape.I;
  a.E = shape.E;
  a.k = shape.k;
  a.has_shared = has_shared;
  a.act_mxfp4 = precision == MOE_ACT_MXFP4;
  if (rp == MOE_PATH_GEMM) return cuda_status(launch_ffn_gemm(a, gemm_buffers(ws, L, shape.E), s));
  a.xh = at<uint16_t>(ws, L.xh);
  a.xexp = at<uint8_t>(ws, L.xexp);
  const bool lane = shape.T <= kLaneMaxT;
  e = launch_x_f16(x, shape.T, shape.H, a.act_mxfp4, at<uint16_t>(ws, L.xh), at<uint8_t>(ws, L.xexp),
                   lane ? at<uint32_t>(ws, L.lane_cnt) : nullptr,
                   lane ? int(lane_cnt_words(shape, has_shared)) : 0, s);
  if (e != cudaSuccess) return cuda_status(e);
  return cuda_status(launch_gemv_path(a, ws, L, s));
}

moe_status_t moe_combine(const float* partial, const float* topk_w, moe_shape_t shape,
                         int32_t has_shared, uint16_t* y, void* stream) {
  moe_status_t st = check_shape(shape);
  if (st != MOE_OK) return st;
  st = check_ptrs({partial, topk_w, y});
  if (st != MOE_OK) return st;
  return cuda_status(launch_combine(partial, topk_w, shape.T, shape.H, shape.k, has_shared != 0,
                                    y, static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_combine_range(const float* partial, const float* topk_w, const int32_t* topk_idx,
                               int32_t e_begin, int32_t e_end, moe_shape_t shape,
                               int32_t has_shared, float* y_f32, void* stream) {
  moe_status_t st = check_shape(shape);
  if (st != MOE_OK) return st;
  st = check_ptrs({partial, topk_w, topk_idx, y_f32});
  if (st != MOE_OK) return st;
  if (e_begin < 0 || e_end < e_begin || e_end > shape.E) return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_combine_range(partial, topk_w, topk_idx, e_begin, e_end, shape.T,
                                          shape.H, shape.k, has_shared != 0, y_f32,
                                          static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_round_bf16(const float* in, int64_t n, uint16_t* out, void* stream) {
  if (n < 0 || n % 4) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (n == 0) return MOE_OK;
  moe_status_t st = check_ptrs({in, out});
  if (st != MOE_OK) return st;
  return cuda_status(launch_round_bf16(in, n, out, static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_layer_forward(const uint16_t* x, const float* w_router, const float* bias,
                               const moe_mxfp4_experts_t* experts,
                               const moe_mxfp4_experts_t* shared, moe_shape_t shape,
                               int32_t path, int32_t precision, uint16_t* y,
                               int32_t* topk_idx_out, float* topk_w_out, void* ws,
                               size_t ws_bytes, void* stream) {
  moe_status_t st = check_shape(shape);
  if (st != MOE_OK) return st;
  if (!valid_path(path) || !valid_precision(precision)) return MOE_ERR_INVALID_ARG;
  st = check_experts(experts, shape.E);
  if (st != MOE_OK) return st;
  if (shared && (st = check_experts(shared, 1)) != MOE_OK) return st;
  st = check_ptrs({x, w_router, y, ws});
  if (st != MOE_OK) return st;
  if (!opt_ok(bias) || !opt_ok(topk_idx_out) || !opt_ok(topk_w_out)) return MOE_ERR_INVALID_ARG;
  const int rp = resolve_path(path, precision, shape);
  if (rp < 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  const int has_shared = shared != nullptr;
  const WsLayout L = ws_layout(shape, has_shared, rp == MOE_PATH_GEMM);
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  RouteArgs r{};
  r.x = x;
  r.w_router = w_router;
  r.bias = bias;
  r.logits = at<float>(ws, L.logits);
  r.idx = topk_idx_out ? topk_idx_out : at<int32_t>(ws, L.idx);
  r.w = topk_w_out ? topk_w_out : at<float>(ws, L.w);
  r.counts = at<int32_t>(ws, L.counts);
  r.offsets = at<int32_t>(ws, L.offsets);
  r.entries = at<int32_t>(ws, L.entries);
  r.plan = at<int32_t>(ws, L.plan);
  r.counter = at<uint32_t>(ws, L.counters);
  r.err = at<int>(ws, L.err);
  r.T = shape.T;
  r.H = shape.H;
  r.E = shape.E;
  r.k = shape.k;
  // the h / partial regions are free until the expert FFNs: the router's
  // K-split sums and the bucket's per-chunk counts
  r.lpart = at<float>(ws, L.h);
  r.lpart_bytes = L.total - L.h;
  if (rp == MOE_PATH_GEMV) {
    r.xh = at<uint16_t>(ws, L.xh);
    r.xexp = at<uint8_t>(ws, L.xexp);
    r.act_mxfp4 = precision == MOE_ACT_MXFP4;
    if (shape.T <= kLaneMaxT) {
      r.cnt_clear = at<uint32_t>(ws, L.lane_cnt);
      r.cnt_words = int(lane_cnt_words(shape, has_shared));
    }
  }
  r.has_shared = has_shared;
  cudaError_t e;
  if (shape.T <= kFusedRouteMaxT) {
    e = launch_route_logits(r, true, s);
  } else {
    e = launch_route_logits(r, false, s);
    if (e == cudaSuccess) e = launch_topk(r, s);
    if (e == cudaSuccess) e = launch_bucket(r, s);
    if (e == cudaSuccess && r.xh != nullptr)
      e = launch_x_f16(x, shape.T, shape.H, r.act_mxfp4, r.xh, r.xexp, r.cnt_clear, r.cnt_words, s);
  }
  if (e != cudaSuccess) return cuda_status(e);

  FfnArgs a{};
  a.ex = ptrs_of(experts);
  a.sh = ptrs_of(shared);
  a.x = x;
  a.offsets = r.offsets;
  a.entries = r.entries;
  a.plan = r.plan;
  a.topk_w = r.w;
  a.h = at<float>(ws, L.h);
  a.partial = at<float>(ws, L.partial);
  a.err = r.err;
  a.T = shape.T;
  a.H = shape.H;
  a.I = shape.I;
  a.E = shape.E;
  a.k = shape.k;
  a.has_shared = has_shared;
  a.act_mxfp4 = precision == MOE_ACT_MXFP4;
  a.xh = r.xh;
  a.xexp = r.xexp;
  e = rp == MOE_PATH_GEMM ? launch_ffn_gemm(a, gemm_buffers(ws, L, shape.E), s)
                          : launch_gemv_path(a, ws, L, s);
  if (e == cudaSuccess)
    e = launch_combine(a.partial, r.w, shape.T, shape.H, shape.k, has_shared, y, s);
  return cuda_status(e);
}

moe_status_t moe_act_quant_mxfp4(const float* in, int32_t rows, int32_t K, uint8_t* q_out,
                                 uint8_t* s_out, void* stream) {
  if (rows < 0 || K < 32 || K % 32) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (rows == 0) return MOE_OK;
  moe_status_t st = check_ptrs({in, q_out});
  if (st != MOE_OK) return st;
  if (s_out == nullptr) return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_act_quant(in, rows, K, q_out, s_out, static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_decode_mxfp4(const uint8_t* q, const uint8_t* s, int32_t rows, int32_t K,
                              float* out, void* stream) {
  if (rows < 0 || K < 32 || K % 32) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (rows == 0) return MOE_OK;
  moe_status_t st = check_ptrs({q, out});
  if (st != MOE_OK) return st;
  if (s == nullptr) return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_decode(q, s, rows, K, out, static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_get_error(void* ws, void* stream) {
  if (ws == nullptr || !aligned16(ws)) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return cuda_status(cudaErrorUnknown);
  int host[2] = {0, 0};
  if (cudaMemcpy(host, ws, sizeof(host), cudaMemcpyDeviceToHost) != cudaSuccess)
    return cuda_status(cudaErrorUnknown);
  if (host[0] != 0 && cudaMemset(ws, 0, sizeof(host)) != cudaSuccess)
    return cuda_status(cudaErrorUnknown);
  return host[0];
}

const char* moe_status_string(moe_status_t status) {
  switch (status) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument (null or misaligned pointer, bad enum)";
    case MOE_ERR_UNSUPPORTED_SHAPE: return "unsupported shape or path";
    case MOE_ERR_WORKSPACE: return "workspace too small";
    case MOE_ERR_CUDA: return "CUDA launch or runtime error";
    case MOE_ERR_TIMEOUT: return "device-side wait gave up";
    case MOE_ERR_DEVICE_DATA: return "invalid data found on the device (expert index, offsets)";
    default: return "unknown status";
  }
}

const char* moe_version(void) { return "0.1.0"; }

}  // extern "C"
