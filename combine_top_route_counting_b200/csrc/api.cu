// C ABI of the library: argument checks, workspace layout, and the
// orchestration of the layer's steps on one stream. See include/moe.h for the
// contract of every entry point.
#include <atomic>
#include <mutex>

#include "internal.cuh"

namespace moe {

namespace {
std::atomic<int64_t> g_launches{0};

constexpr size_t kAlign = 1024;
inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

moe_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_CUDA_ERROR; }

// Basic shape limits shared by every entry point.
moe_status_t check_shape(const moe_shape_t* s) {
  if (!s) return MOE_INVALID_ARG;
  if (s->P < 1 || s->P > 64 || s->N < 0 || s->E < 1 || s->E > 1024 || s->k < 1 || s->k > 16 ||
      s->k > s->E || s->pad < 1 || s->pad > (1 << 16))
    return MOE_UNSUPPORTED_SHAPE;
  const int64_t routes = static_cast<int64_t>(s->P) * s->N * s->k;
  const int64_t rows = routes + static_cast<int64_t>(s->E) * (s->pad - 1) + 255;
  if (routes >= (int64_t{1} << 31) || rows >= (int64_t{1} << 31)) return MOE_UNSUPPORTED_SHAPE;
  return MOE_OK;
}

// Extra limits of the expert FFN (tcgen05 tiles of 128 rows x 256 columns,
// K steps of 64, TMA coordinates in int32).
moe_status_t check_ffn_shape(const moe_shape_t* s) {
  moe_status_t st = check_shape(s);
  if (st != MOE_OK) return st;
  if (s->H < 256 || s->H % 256 != 0 || s->I < 128 || s->I % 128 != 0 || s->pad % 128 != 0)
    return MOE_UNSUPPORTED_SHAPE;
  if (static_cast<int64_t>(s->E) * s->H >= (int64_t{1} << 31) ||
      static_cast<int64_t>(s->E) * s->I >= (int64_t{1} << 31))
    return MOE_UNSUPPORTED_SHAPE;
  return MOE_OK;
}

int64_t rows_max_of(const moe_shape_t* s) {
  const int64_t raw =
      static_cast<int64_t>(s->P) * s->N * s->k + static_cast<int64_t>(s->E) * (s->pad - 1);
  return (raw + 255) / 256 * 256;
}

// Layout of the layer workspace (offsets in bytes, each kAlign-aligned).
struct LayerWs {
  size_t ids, gates, route_row, phi, offsets, counts, sched, xg, h, y, total;
  size_t logits, x, out, total_host;  // moe_layer_forward_host additions
};

LayerWs layer_ws(const moe_shape_t* s) {
  LayerWs w{};
  const size_t routes = static_cast<size_t>(s->P) * s->N * s->k;
  const size_t rows = static_cast<size_t>(rows_max_of(s));
  const size_t tokens = static_cast<size_t>(s->P) * s->N;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = align_up(o + (bytes ? bytes : 1), kAlign);
    return at;
  };
  w.ids = take(routes * 4);
  w.gates = take(routes * 4);
  w.route_row = take(routes * 4);
  w.phi = take(rows * 8);
  w.offsets = take((s->E + 1) * 4);
  w.counts = take(static_cast<size_t>(s->E) * s->P * 4);
  w.sched = take(schedule_ws_bytes(s->P, s->N, s->k, s->E));
  w.xg = take(rows * s->H * 2);
  w.h = take(rows * s->I * 2);
  w.y = take(rows * s->H * 4);
  w.total = o;
  w.logits = take(tokens * s->E * 4);
  w.x = take(tokens * s->H * 2);
  w.out = take(tokens * s->H * 2);
  w.total_host = o;
  return w;
}

template <class T>
T* at(void* base, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(base) + off);
}

}  // namespace

void note_launches(int64_t n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

int device_sm_count() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

namespace {

// The layer body on device buffers (shared by both layer entry points).
moe_status_t layer_body(const float* logits, const uint16_t* x, const uint16_t* W1,
                        const uint16_t* W3, const uint16_t* W2, uint16_t* out,
                        int32_t minibatch_tokens, void* ws, int32_t* dev_status,
                        const moe_shape_t* sh, cudaStream_t s, void* const* ev) {
  const LayerWs w = layer_ws(sh);
  const int64_t rows_max = rows_max_of(sh);
  int32_t* ids = at<int32_t>(ws, w.ids);
  float* gates = at<float>(ws, w.gates);
  int32_t* route_row = at<int32_t>(ws, w.route_row);
  int32_t* phi = at<int32_t>(ws, w.phi);
  int32_t* offsets = at<int32_t>(ws, w.offsets);
  int32_t* counts = at<int32_t>(ws, w.counts);
  int32_t* sched = at<int32_t>(ws, w.sched);
  uint16_t* xg = at<uint16_t>(ws, w.xg);
  uint16_t* h = at<uint16_t>(ws, w.h);
  float* y = at<float>(ws, w.y);

  const int32_t N = sh->N;
  const int32_t T = (minibatch_tokens <= 0 || minibatch_tokens >= N) ? N : minibatch_tokens;
  const bool single = (T == N);
  auto rec = [&](int i) -> cudaError_t {
    if (!ev || !single || !ev[i]) return cudaSuccess;
    return cudaEventRecord(static_cast<cudaEvent_t>(ev[i]), s);
  };

  cudaError_t e = rec(0);
  if (e == cudaSuccess)
    e = launch_route_topk(logits, ids, gates, static_cast<int64_t>(sh->P) * N, sh->E, sh->k, s);
  if (e != cudaSuccess) return from_cuda(e);
  if (N == 0) {
    rec(1);
    rec(2);
    rec(3);
    rec(4);
    rec(5);
    return from_cuda(rec(6));
  }
  for (int32_t t0 = 0; t0 < N; t0 += T) {
    const Slice sl{t0, (N - t0) < T ? (N - t0) : T};
    if ((e = rec(1)) != cudaSuccess) break;
    if ((e = launch_schedule(ids, *sh, sl, phi, offsets, counts, route_row, sched, dev_status, s)) !=
        cudaSuccess)
      break;
    if ((e = rec(2)) != cudaSuccess) break;
    if ((e = launch_dispatch(x, phi, offsets, xg, *sh, rows_max, dev_status, s)) != cudaSuccess)
      break;
    if ((e = rec(3)) != cudaSuccess) break;
    cudaEvent_t mid = (ev && single) ? static_cast<cudaEvent_t>(ev[4]) : nullptr;
    if ((e = launch_expert_ffn(xg, W1, W3, W2, offsets, counts, h, y, *sh, rows_max, dev_status, s,
                               mid)) != cudaSuccess)
      break;
    if ((e = rec(5)) != cudaSuccess) break;
    if ((e = launch_combine(y, route_row, gates, out, *sh, sl, rows_max, dev_status, s)) !=
        cudaSuccess)
      break;
    if ((e = rec(6)) != cudaSuccess) break;
  }
  return from_cuda(e);
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

const char* moe_status_string(moe_status_t st) {
  switch (st) {
    case MOE_OK: return "MOE_OK";
    case MOE_INVALID_ARG: return "MOE_INVALID_ARG";
    case MOE_UNSUPPORTED_SHAPE: return "MOE_UNSUPPORTED_SHAPE";
    case MOE_WORKSPACE_TOO_SMALL: return "MOE_WORKSPACE_TOO_SMALL";
    case MOE_CUDA_ERROR: return "MOE_CUDA_ERROR";
    case MOE_DEVICE_TIMEOUT: return "MOE_DEVICE_TIMEOUT";
    case MOE_BAD_EXPERT_ID: return "MOE_BAD_EXPERT_ID";
    case MOE_BAD_SCHEDULE: return "MOE_BAD_SCHEDULE";
    default: return "MOE_UNKNOWN_STATUS";
  }
}

moe_status_t moe_status_from_device_flags(int32_t flags) {
  if (flags & MOE_DEV_TIMEOUT) return MOE_DEVICE_TIMEOUT;
  if (flags & MOE_DEV_BAD_SCHEDULE) return MOE_BAD_SCHEDULE;
  if (flags & MOE_DEV_BAD_EXPERT_ID) return MOE_BAD_EXPERT_ID;
  return MOE_OK;
}

int64_t moe_rows_max(const moe_shape_t* shape) {
  if (check_shape(shape) != MOE_OK) return -1;
  return rows_max_of(shape);
}

size_t moe_schedule_workspace_bytes(const moe_shape_t* shape) {
  if (check_shape(shape) != MOE_OK) return 0;
  return schedule_ws_bytes(shape->P, shape->N, shape->k, shape->E);
}

size_t moe_layer_workspace_bytes(const moe_shape_t* shape) {
  if (check_ffn_shape(shape) != MOE_OK) return 0;
  return layer_ws(shape).total;
}

size_t moe_layer_host_workspace_bytes(const moe_shape_t* shape) {
  if (check_ffn_shape(shape) != MOE_OK) return 0;
  return layer_ws(shape).total_host;
}

moe_status_t moe_route_topk(const float* logits, int32_t* ids, float* gates,
                            const moe_shape_t* shape, void* stream) {
  moe_status_t st = check_shape(shape);
  if (st != MOE_OK) return st;
  const int64_t n = static_cast<int64_t>(shape->P) * shape->N;
  if (n > 0 && (!logits || !ids || !gates)) return MOE_INVALID_ARG;
  if (!aligned16(logits) || !aligned16(ids) || !aligned16(gates)) return MOE_INVALID_ARG;
  return from_cuda(launch_route_topk(logits, ids, gates, n, shape->E, shape->k,
                                     static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_schedule(const int32_t* ids, int32_t* phi, int32_t* offsets, int32_t* counts,
                          int32_t* route_row, void* ws, size_t ws_bytes, int32_t* dev_status,
                          const moe_shape_t* shape, void* stream) {
  moe_status_t st = check_shape(shape);
  if (st != MOE_OK) return st;
  if (!phi || !offsets || !counts || !dev_status || !ws) return MOE_INVALID_ARG;
  if (shape->N > 0 && (!ids || !route_row)) return MOE_INVALID_ARG;
  if (!aligned16(ids) || !aligned16(phi) || !aligned16(route_row) || !aligned16(ws))
    return MOE_INVALID_ARG;
  if (ws_bytes < schedule_ws_bytes(shape->P, shape->N, shape->k, shape->E))
    return MOE_WORKSPACE_TOO_SMALL;
  return from_cuda(launch_schedule(ids, *shape, Slice{0, shape->N}, phi, offsets, counts,
                                   route_row, static_cast<int32_t*>(ws), dev_status,
                                   static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_dispatch(const uint16_t* x, const int32_t* phi, const int32_t* offsets,
                          uint16_t* xg, int32_t* dev_status, const moe_shape_t* shape,
                          void* stream) {
  moe_status_t st = check_shape(shape);
  if (st != MOE_OK) return st;
  if (shape->H < 8 || shape->H % 8 != 0) return MOE_UNSUPPORTED_SHAPE;
  if (!phi || !offsets || !xg || !dev_status || (shape->N > 0 && !x)) return MOE_INVALID_ARG;
  if (!aligned16(x) || !aligned16(phi) || !aligned16(xg)) return MOE_INVALID_ARG;
  return from_cuda(launch_dispatch(x, phi, offsets, xg, *shape, rows_max_of(shape), dev_status,
                                   static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_expert_ffn(const uint16_t* xg, const uint16_t* W1, const uint16_t* W3,
                            const uint16_t* W2, const int32_t* offsets, const int32_t* counts,
                            uint16_t* h, float* y, int32_t* dev_status, const moe_shape_t* shape,
                            void* stream) {
  moe_status_t st = check_ffn_shape(shape);
  if (st != MOE_OK) return st;
  if (!xg || !W1 || !W3 || !W2 || !offsets || !h || !y || !dev_status) return MOE_INVALID_ARG;
  if (!aligned16(xg) || !aligned16(W1) || !aligned16(W3) || !aligned16(W2) || !aligned16(h) ||
      !aligned16(y))
    return MOE_INVALID_ARG;
  return from_cuda(launch_expert_ffn(xg, W1, W3, W2, offsets, counts, h, y, *shape,
                                     rows_max_of(shape), dev_status,
                                     static_cast<cudaStream_t>(stream), nullptr));
}

moe_status_t moe_combine(const float* y, const int32_t* route_row, const float* gates,
                         uint16_t* out, int32_t* dev_status, const moe_shape_t* shape,
                         void* stream) {
  moe_status_t st = check_shape(shape);
  if (st != MOE_OK) return st;
  if (shape->H < 4 || shape->H % 4 != 0) return MOE_UNSUPPORTED_SHAPE;
  if (!dev_status || (shape->N > 0 && (!y || !route_row || !gates || !out)))
    return MOE_INVALID_ARG;
  if (!aligned16(y) || !aligned16(out)) return MOE_INVALID_ARG;
  return from_cuda(launch_combine(y, route_row, gates, out, *shape, Slice{0, shape->N},
                                  rows_max_of(shape), dev_status,
                                  static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_layer_forward(const float* logits, const uint16_t* x, const uint16_t* W1,
                               const uint16_t* W3, const uint16_t* W2, uint16_t* out,
                               int32_t minibatch_tokens, void* ws, size_t ws_bytes,
                               int32_t* dev_status, const moe_shape_t* shape, void* stream,
                               void* const* stage_events) {
  moe_status_t st = check_ffn_shape(shape);
  if (st != MOE_OK) return st;
  if (!W1 || !W3 || !W2 || !ws || !dev_status || (shape->N > 0 && (!logits || !x || !out)))
    return MOE_INVALID_ARG;
  if (!aligned16(logits) || !aligned16(x) || !aligned16(W1) || !aligned16(W3) || !aligned16(W2) ||
      !aligned16(out) || !aligned16(ws))
    return MOE_INVALID_ARG;
  if (minibatch_tokens < 0) return MOE_INVALID_ARG;
  if (ws_bytes < layer_ws(shape).total) return MOE_WORKSPACE_TOO_SMALL;
  return layer_body(logits, x, W1, W3, W2, out, minibatch_tokens, ws, dev_status, shape,
                    static_cast<cudaStream_t>(stream), stage_events);
}

moe_status_t moe_layer_forward_host(const float* logits_host, const uint16_t* x_host,
                                    const uint16_t* W1, const uint16_t* W3, const uint16_t* W2,
                                    uint16_t* out_host, int32_t minibatch_tokens, void* ws,
                                    size_t ws_bytes, int32_t* dev_status,
                                    const moe_shape_t* shape, void* stream) {
  moe_status_t st = check_ffn_shape(shape);
  if (st != MOE_OK) return st;
  if (!W1 || !W3 || !W2 || !ws || !dev_status ||
      (shape->N > 0 && (!logits_host || !x_host || !out_host)))
    return MOE_INVALID_ARG;
  if (!aligned16(W1) || !aligned16(W3) || !aligned16(W2) || !aligned16(ws))
    return MOE_INVALID_ARG;
  if (minibatch_tokens < 0) return MOE_INVALID_ARG;
  const LayerWs w = layer_ws(shape);
  if (ws_bytes < w.total_host) return MOE_WORKSPACE_TOO_SMALL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t tokens = static_cast<size_t>(shape->P) * shape->N;
  float* logits = at<float>(ws, w.logits);
  uint16_t* x = at<uint16_t>(ws, w.x);
  uint16_t* out = at<uint16_t>(ws, w.out);
  cudaError_t e = cudaMemcpyAsync(logits, logits_host, tokens * shape->E * 4,
                                  cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(x, x_host, tokens * shape->H * 2, cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return MOE_CUDA_ERROR;
  st = layer_body(logits, x, W1, W3, W2, out, minibatch_tokens, ws, dev_status, shape, s, nullptr);
  if (st != MOE_OK) return st;
  e = cudaMemcpyAsync(out_host, out, tokens * shape->H * 2, cudaMemcpyDeviceToHost, s);
  return from_cuda(e);
}

int64_t moe_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

moe_status_t moe_selftest_bounded_wait(int32_t* dev_status, int64_t timeout_ns, void* stream) {
  if (!dev_status || timeout_ns <= 0) return MOE_INVALID_ARG;
  return from_cuda(launch_selftest_wait(dev_status, timeout_ns, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
