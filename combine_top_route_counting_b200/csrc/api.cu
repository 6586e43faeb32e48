// C ABI of the library: argument checks, workspace layout, and the
// orchestration of the layer's steps on one stream. See include/moe.h for the
// contract of every entry point.
#include <atomic>
#include <mutex>

#include "internal.cuh"

namespace moe {

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

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

namespace {
std::atomic<int64_t> g_launches{0};

constexpr size_t kAlign = 1024;
inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Buffers written with 32-byte vector stores.
bool aligned32(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }

moe_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_CUDA_ERROR; }

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

// Extra limits of the backward pass (CTA-pair tiles of 256 rows x 256 columns
// in every GEMM: segments padded to multiples of 256, I a multiple of 256).
moe_status_t check_bwd_shape(const moe_shape_t* s) {
  moe_status_t st = check_ffn_shape(s);
  if (st != MOE_OK) return st;
  if (s->I % 256 != 0 || s->pad % 256 != 0) return MOE_UNSUPPORTED_SHAPE;
  return MOE_OK;
}

// Extra limits of the MXFP8 expert FFN (block-scaled CTA-pair tiles of 256
// rows; GEMM1 output blocks of 128 h columns, GEMM2 of 256 y columns; 128 K
// values per pipeline stage).
moe_status_t check_mx_shape(const moe_shape_t* s) {
  moe_status_t st = check_ffn_shape(s);
  if (st != MOE_OK) return st;
  if (s->pad % 256 != 0) return MOE_UNSUPPORTED_SHAPE;
  // scale-atom indices of the TMA loads are int32
  const int64_t atoms_w = static_cast<int64_t>(s->E) * (s->I / 128) * (s->H / 128);
  const int64_t atoms_x = rows_max_of(s) / 128 * (s->H / 128);
  if (atoms_w >= (int64_t{1} << 31) || atoms_x >= (int64_t{1} << 31)) return MOE_UNSUPPORTED_SHAPE;
  return MOE_OK;
}

// Layout of the layer workspace (offsets in bytes, each kAlign-aligned).
// The training layout keeps what the backward reads (ids, gates, route_row,
// Phi, offsets, counts, xg, h and the pre-activations ab) and adds the
// backward's buffers; dxg [rows, H] fp32 reuses y, which is dead once the
// forward's combine has run.
struct LayerWs {
  size_t ids, gates, route_row, phi, offsets, counts, sched, ctr, xg, h, y, total;
  size_t logits[2], x[2], out[2], total_host;  // moe_layer_forward_host additions
  size_t ab, dys, dab, hg, gate_row, part, total_train;  // training additions
  size_t sh_off, sh_x, sh_h, sh_y, total_mx;  // the MXFP8 layer's shared expert
};

LayerWs layer_ws(const moe_shape_t* s) {
  LayerWs w{};
  const size_t routes = static_cast<size_t>(s->P) * s->N * s->k;
  const size_t rows = static_cast<size_t>(rows_max_of(s));
  const size_t tokens = static_cast<size_t>(s->P) * s->N;
  size_t o = 0;
  auto take = [](size_t& cur, size_t bytes) {
    const size_t at = cur;
    cur = align_up(cur + (bytes ? bytes : 1), kAlign);
    return at;
  };
  w.ids = take(o, routes * 4);
  w.gates = take(o, routes * 4);
  w.route_row = take(o, routes * 4);
  w.phi = take(o, rows * 8);
  w.offsets = take(o, (s->E + 1) * 4);
  w.counts = take(o, static_cast<size_t>(s->E) * s->P * 4);
  w.sched = take(o, schedule_ws_bytes(s->P, s->N, s->k, s->E));
  // the GEMMs' tile counter (words 0-1), the fused dispatch's next block
  // (word 16) and ready flags (words 32..), zeroed at the start of each call
  w.ctr = take(o, (32 + rows / 128) * 4);
  w.xg = take(o, rows * s->H * 2);
  w.h = take(o, rows * s->I * 2);
  w.y = take(o, rows * s->H * 4);
  w.total = o;
  size_t oh = o;
  for (int b = 0; b < 2; ++b) {  // consecutive host-buffer calls alternate
    w.logits[b] = take(oh, tokens * s->E * 4);
    w.x[b] = take(oh, tokens * s->H * 2);
    w.out[b] = take(oh, tokens * s->H * 2);
  }
  w.total_host = oh;
  size_t ot = o;
  w.ab = take(ot, rows * s->I * 4);
  w.dys = take(ot, rows * s->H * 2);
  w.dab = take(ot, rows * s->I * 4);
  w.hg = take(ot, rows * s->I * 2);
  w.gate_row = take(ot, rows * 4);
  w.part = take(ot, rows * (s->I / 128) * 4);
  w.total_train = ot;
  size_t om = o;
  const size_t tok_rows = (tokens + 255) / 256 * 256;
  w.sh_off = take(om, 8);
  w.sh_x = take(om, tokens % 256 ? tok_rows * s->H * 2 : 0);  // padded copy of x, ragged only
  w.sh_h = take(om, tok_rows * s->I * 2);
  w.sh_y = take(om, tok_rows * s->H * 4);
  w.total_mx = om;
  return w;
}

template <class T>
T* at(void* base, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(base) + off);
}

}  // namespace

void note_launches(int64_t n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

int device_sm_count() {
  static std::atomic<int> cache[64];  // 0 = not looked up yet
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  int n = cache[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cache[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

namespace {

struct LayerBufs {
  int32_t *ids, *route_row, *phi, *offsets, *counts, *sched;
  int *ctr, *land;
  float *gates, *y;
  uint16_t *xg, *h;
};

LayerBufs layer_bufs(void* ws, const LayerWs& w) {
  LayerBufs b;
  b.ids = at<int32_t>(ws, w.ids);
  b.gates = at<float>(ws, w.gates);
  b.route_row = at<int32_t>(ws, w.route_row);
  b.phi = at<int32_t>(ws, w.phi);
  b.offsets = at<int32_t>(ws, w.offsets);
  b.counts = at<int32_t>(ws, w.counts);
  b.sched = at<int32_t>(ws, w.sched);
  b.ctr = at<int>(ws, w.ctr);
  b.land = b.ctr + 16;
  b.xg = at<uint16_t>(ws, w.xg);
  b.h = at<uint16_t>(ws, w.h);
  b.y = at<float>(ws, w.y);
  return b;
}

// The scratch words a layer call's kernels expect at zero when it starts: the
// tile counter and landing words, and the schedule's barrier and totals. The
// routing kernel zeroes them (first slice); later slices zero what they reuse.
ZeroSpec call_zeroes(const LayerBufs& b, const moe_shape_t* sh) {
  return ZeroSpec{b.ctr, static_cast<int32_t>(32 + rows_max_of(sh) / 128),
                  schedule_barrier_word(b.sched, *sh), schedule_zero_words(*sh)};
}

// Schedule -> dispatch -> FFN -> combine for one token slice (steps 2-4).
// ev (7 events, may be null) marks the stage boundaries 1..6.
// ab (training, whole batch only): GEMM1 also keeps the pre-activations.
// first: the call's first slice, whose scratch words the routing kernel
// zeroed (later slices zero the landing words and the schedule's barrier and
// totals themselves).
cudaError_t run_slice(const LayerBufs& b, const uint16_t* x, const uint16_t* W1, const uint16_t* W3,
                      const uint16_t* W2, uint16_t* out, Slice sl, const moe_shape_t* sh,
                      int32_t* dev_status, cudaStream_t s, void* const* ev, bool first,
                      uint16_t* ab = nullptr) {
  const int64_t rows_max = rows_max_of(sh);
  auto rec = [&](int i) -> cudaError_t {
    return (ev && ev[i]) ? cudaEventRecord(static_cast<cudaEvent_t>(ev[i]), s) : cudaSuccess;
  };
  cudaError_t e;
  if ((e = rec(1)) != cudaSuccess) return e;
  if ((e = launch_schedule(b.ids, *sh, sl, b.phi, b.offsets, b.counts, b.route_row, b.sched,
                           dev_status, s, first)) != cudaSuccess)
    return e;
  // With CTA-pair tiles (segments padded to 256 rows) the pull dispatch runs
  // inside GEMM1: its spare warp lands the rows into xg block by block while
  // the tensor cores work on the blocks already there. Otherwise the dispatch
  // is its own HBM-bound gather before the FFN. (Feeding the MMAs straight
  // from x by row gathers, moe_expert_ffn_gather, measured 2.6-3x slower.)
  if ((e = rec(2)) != cudaSuccess) return e;
  const bool fused = sh->pad % 256 == 0;
  const LandArgs land{x, b.phi, b.land, b.land + 16};
  if (fused) {
    if (!first &&
        (e = cudaMemsetAsync(b.land, 0, (16 + rows_max / 128) * sizeof(int), s)) != cudaSuccess)
      return e;
  } else if ((e = launch_dispatch(x, b.phi, b.offsets, b.xg, *sh, rows_max, dev_status, s)) !=
             cudaSuccess) {
    return e;
  }
  if ((e = rec(3)) != cudaSuccess) return e;
  cudaEvent_t mid = (ev && ev[4]) ? static_cast<cudaEvent_t>(ev[4]) : nullptr;
  if ((e = launch_expert_ffn(b.xg, W1, W3, W2, b.offsets, b.counts, b.h, b.y, *sh, rows_max,
                             dev_status, s, mid, ab, b.ctr, fused ? &land : nullptr)) !=
      cudaSuccess)
    return e;
  if ((e = rec(5)) != cudaSuccess) return e;
  if ((e = launch_combine(b.y, b.route_row, b.gates, out, *sh, sl, rows_max, dev_status, s)) !=
      cudaSuccess)
    return e;
  return rec(6);
}

// The layer body on device buffers (shared by both layer entry points).
moe_status_t layer_body(const float* logits, const uint16_t* x, const uint16_t* W1,
                        const uint16_t* W3, const uint16_t* W2, uint16_t* out,
                        int32_t minibatch_tokens, void* ws, int32_t* dev_status,
                        const moe_shape_t* sh, cudaStream_t s, void* const* ev,
                        bool train = false) {
  const LayerWs lw = layer_ws(sh);
  const LayerBufs b = layer_bufs(ws, lw);
  uint16_t* ab = train ? at<uint16_t>(ws, lw.ab) : nullptr;
  if (train) minibatch_tokens = 0;  // one schedule over the whole batch, kept for the backward
  const int32_t N = sh->N;
  const int32_t T = (minibatch_tokens <= 0 || minibatch_tokens >= N) ? N : minibatch_tokens;
  void* const* ev_use = (T == N) ? ev : nullptr;  // stage events: single-slice runs only
  cudaError_t e = (ev_use && ev_use[0]) ? cudaEventRecord(static_cast<cudaEvent_t>(ev_use[0]), s)
                                        : cudaSuccess;
  const ZeroSpec z = call_zeroes(b, sh);
  if (e == cudaSuccess)
    e = launch_route_topk(logits, b.ids, b.gates, static_cast<int64_t>(sh->P) * N, sh->E, sh->k, s,
                          &z);
  if (e != cudaSuccess) return from_cuda(e);
  if (N == 0) {
    for (int i = 1; i < 7 && ev_use; ++i)
      if (ev_use[i]) cudaEventRecord(static_cast<cudaEvent_t>(ev_use[i]), s);
    return MOE_OK;
  }
  for (int32_t t0 = 0; t0 < N && e == cudaSuccess; t0 += T) {
    const Slice sl{t0, (N - t0) < T ? (N - t0) : T};
    e = run_slice(b, x, W1, W3, W2, out, sl, sh, dev_status, s, ev_use, t0 == 0, ab);
  }
  return from_cuda(e);
}

// The MXFP8 layer on device buffers. It uses the bf16 layer's workspace: the
// E4M3 codes and tiled scales of the gathered tokens fill the xg region
// (rows*H + rows*H/32 bytes of rows*H*2), those of h the h region.
// ev (7 events, may be null) as moe_layer_forward.
cudaError_t layer_body_mx(const float* logits, const uint16_t* x, const uint8_t* W1q,
                          const uint8_t* W1s, const uint8_t* W3q, const uint8_t* W3s,
                          const uint8_t* W2q, const uint8_t* W2s, const uint16_t* Ws1,
                          const uint16_t* Ws3, const uint16_t* Ws2, uint16_t* out, void* ws,
                          int32_t* dev_status, const moe_shape_t* sh, cudaStream_t s,
                          void* const* ev) {
  const LayerWs w = layer_ws(sh);
  const LayerBufs b = layer_bufs(ws, w);
  const int64_t rows_max = rows_max_of(sh);
  uint8_t* xq = at<uint8_t>(ws, w.xg);
  uint8_t* xs = xq + static_cast<size_t>(rows_max) * sh->H;
  uint8_t* hq = at<uint8_t>(ws, w.h);
  uint8_t* hs = hq + static_cast<size_t>(rows_max) * sh->I;
  auto rec = [&](int i) -> cudaError_t {
    return (ev && ev[i]) ? cudaEventRecord(static_cast<cudaEvent_t>(ev[i]), s) : cudaSuccess;
  };
  cudaError_t e;
  if ((e = rec(0)) != cudaSuccess) return e;
  const ZeroSpec z = call_zeroes(b, sh);
  if ((e = launch_route_topk(logits, b.ids, b.gates, static_cast<int64_t>(sh->P) * sh->N, sh->E,
                             sh->k, s, &z)) != cudaSuccess)
    return e;
  if (sh->N == 0) {
    for (int i = 1; i < 7; ++i)
      if ((e = rec(i)) != cudaSuccess) return e;
    return cudaSuccess;
  }
  if ((e = rec(1)) != cudaSuccess) return e;
  if ((e = launch_schedule(b.ids, *sh, Slice{0, sh->N}, b.phi, b.offsets, b.counts, b.route_row,
                           b.sched, dev_status, s, /*barrier_zeroed=*/true)) != cudaSuccess)
    return e;
  if ((e = rec(2)) != cudaSuccess) return e;
  // the quantising pull dispatch lands inside GEMM1 (its spare warp writes
  // the codes and tiled scales of 128-row blocks as the tensor cores consume
  // earlier ones); the landing words were zeroed by the routing kernel
  const LandArgs land{x, b.phi, b.land, b.land + 16};
  if ((e = rec(3)) != cudaSuccess) return e;
  // the bf16 shared expert over every token (its time counts in stage 3, the
  // routed GEMM1's); nothing on one GPU to overlap it with
  float* ys = nullptr;
  if (Ws1) {
    ys = at<float>(ws, w.sh_y);
    if ((e = launch_dense_ffn(x, static_cast<int64_t>(sh->P) * sh->N, Ws1, Ws3, Ws2,
                              at<uint16_t>(ws, w.sh_x), at<uint16_t>(ws, w.sh_h), ys,
                              at<int32_t>(ws, w.sh_off), sh->H,
                              sh->I, dev_status, s, b.ctr)) != cudaSuccess)
      return e;
  }
  cudaEvent_t mid = ev ? static_cast<cudaEvent_t>(ev[4]) : nullptr;
  if ((e = launch_expert_ffn_mxfp8(xq, xs, W1q, W1s, W3q, W3s, W2q, W2s, b.offsets, b.counts, hq,
                                   hs, b.y, *sh, rows_max, dev_status, s, mid, b.ctr, &land)) !=
      cudaSuccess)
    return e;
  if ((e = rec(5)) != cudaSuccess) return e;
  if ((e = launch_combine(b.y, b.route_row, b.gates, out, *sh, Slice{0, sh->N}, rows_max,
                          dev_status, s, ys)) != cudaSuccess)
    return e;
  return rec(6);
}

// The backward pass on the state a training forward left in `ws`.
// ev (8 events, may be null): start, then after the reverse combine, the
// dh GEMM, the dx GEMM, the reverse dispatch, the router gradient, dW2 and
// dW1 | dW3.
cudaError_t backward_body(const uint16_t* dout, const uint16_t* W1, const uint16_t* W3,
                          const uint16_t* W2, uint16_t* dx, float* dlogits, float* dW1, float* dW3,
                          float* dW2, void* ws, int32_t* dev_status, const moe_shape_t* sh,
                          cudaStream_t s, void* const* ev) {
  const LayerWs w = layer_ws(sh);
  const LayerBufs b = layer_bufs(ws, w);
  const int64_t rows_max = rows_max_of(sh);
  uint16_t* ab = at<uint16_t>(ws, w.ab);
  uint16_t* dys = at<uint16_t>(ws, w.dys);
  uint16_t* dab = at<uint16_t>(ws, w.dab);
  uint16_t* hg = at<uint16_t>(ws, w.hg);
  float* gate_row = at<float>(ws, w.gate_row);
  float* part = at<float>(ws, w.part);
  float* dxg = b.y;
  auto rec = [&](int i) -> cudaError_t {
    return (ev && ev[i]) ? cudaEventRecord(static_cast<cudaEvent_t>(ev[i]), s) : cudaSuccess;
  };
  auto evt = [&](int i) -> cudaEvent_t { return ev ? static_cast<cudaEvent_t>(ev[i]) : nullptr; };
  cudaError_t e;
  if ((e = rec(0)) != cudaSuccess) return e;
  if (sh->N == 0) {  // no routes: every weight gradient is zero
    const size_t wbytes = static_cast<size_t>(sh->E) * sh->H * sh->I * 4;
    if ((e = cudaMemsetAsync(dW1, 0, wbytes, s)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(dW3, 0, wbytes, s)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(dW2, 0, wbytes, s)) != cudaSuccess) return e;
    for (int i = 1; i < 8; ++i)
      if ((e = rec(i)) != cudaSuccess) return e;
    return cudaSuccess;
  }
  if ((e = cudaMemsetAsync(b.ctr, 0, 8, s)) != cudaSuccess) return e;
  if ((e = launch_reverse_combine(dout, b.phi, b.offsets, b.route_row, b.gates, dys, gate_row, *sh,
                                  rows_max, dev_status, s)) != cudaSuccess)
    return e;
  if ((e = rec(1)) != cudaSuccess) return e;
  if ((e = launch_expert_ffn_dgrad(dys, gate_row, ab, b.h, W1, W3, W2, b.offsets, b.counts, dab, hg,
                                   part, dxg, *sh, rows_max, dev_status, s, evt(2), b.ctr)) !=
      cudaSuccess)
    return e;
  if ((e = rec(3)) != cudaSuccess) return e;
  if ((e = launch_reverse_dispatch(dxg, b.route_row, dx, *sh, rows_max, dev_status, s)) !=
      cudaSuccess)
    return e;
  if ((e = rec(4)) != cudaSuccess) return e;
  if ((e = launch_router_backward(part, sh->I / 128, b.route_row, b.ids, b.gates, dlogits,
                                  static_cast<int64_t>(sh->P) * sh->N, sh->E, sh->k, rows_max,
                                  dev_status, s)) != cudaSuccess)
    return e;
  if ((e = rec(5)) != cudaSuccess) return e;
  // weight gradients last: deferred until every activation gradient is done
  if ((e = launch_expert_ffn_wgrad(b.xg, dys, dab, hg, b.offsets, b.counts, dW1, dW3, dW2, *sh,
                                   rows_max, dev_status, s, evt(6), b.ctr)) != cudaSuccess)
    return e;
  return rec(7);
}

// Per-device copy engines' streams and events of moe_layer_forward_host,
// created on first use and kept until the process exits.
constexpr int kRing = 4;
struct CopyRes {
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaEvent_t lg = nullptr, fin = nullptr;
  cudaEvent_t ex[kRing] = {}, ed[kRing] = {};
  cudaEvent_t in_free[2] = {};   // input buffers of parity b no longer read
  cudaEvent_t out_free[2] = {};  // output buffer of parity b copied out
  uint64_t calls = 0;
  bool ready = false;
};
std::mutex g_copy_mu;
CopyRes g_copy[64];

cudaError_t copy_res(CopyRes** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  CopyRes& r = g_copy[dev];
  if (!r.ready) {
    const unsigned ef = cudaEventDisableTiming;
    if ((e = cudaStreamCreateWithFlags(&r.h2d, cudaStreamNonBlocking)) != cudaSuccess) return e;
    if ((e = cudaStreamCreateWithFlags(&r.d2h, cudaStreamNonBlocking)) != cudaSuccess) return e;
    if ((e = cudaEventCreateWithFlags(&r.in_free[0], ef)) != cudaSuccess) return e;
    if ((e = cudaEventCreateWithFlags(&r.in_free[1], ef)) != cudaSuccess) return e;
    if ((e = cudaEventCreateWithFlags(&r.out_free[0], ef)) != cudaSuccess) return e;
    if ((e = cudaEventCreateWithFlags(&r.out_free[1], ef)) != cudaSuccess) return e;
    if ((e = cudaEventCreateWithFlags(&r.lg, ef)) != cudaSuccess) return e;
    if ((e = cudaEventCreateWithFlags(&r.fin, ef)) != cudaSuccess) return e;
    for (int i = 0; i < kRing; ++i) {
      if ((e = cudaEventCreateWithFlags(&r.ex[i], ef)) != cudaSuccess) return e;
      if ((e = cudaEventCreateWithFlags(&r.ed[i], ef)) != cudaSuccess) return e;
    }
    r.ready = true;
  }
  *out = &r;
  return cudaSuccess;
}

// Host-buffer layer. Consecutive calls alternate between two device copies of
// the inputs and of the output (parity b), so the host-to-device copy of call
// i+1 runs while call i still computes: it only waits until call i-1, the last
// user of the same copies, has finished reading them. Within a call, the rows
// of slice [t0, t0+Tm) of every peer are copied in on the h2d stream while the
// previous slice computes on `s`, and copied out on the d2h stream while the
// next one computes (the transfer minibatch of "Mixture-of-Kittens" notes
// section 3 and "Beyond Peak TFLOPs" section 1: chunk k transfers while chunk
// k-1 computes). Without out_ready, `s` waits for every copy of the call
// before the call ends. With out_ready, `s` does not wait for the copy out
// (the event marks its end), so call i+1 computes while call i's output
// travels; call i+2 writes the same device output copy only after it has
// been copied out.
cudaError_t layer_host_pipeline(const float* logits_host, const uint16_t* x_host,
                                const uint16_t* W1, const uint16_t* W3, const uint16_t* W2,
                                uint16_t* out_host, int32_t minibatch_tokens, void* ws,
                                int32_t* dev_status, const moe_shape_t* sh, cudaStream_t s,
                                cudaEvent_t out_ready) {
  std::lock_guard<std::mutex> lock(g_copy_mu);
  CopyRes* cr = nullptr;
  cudaError_t e = copy_res(&cr);
  if (e != cudaSuccess) return e;
  const int b = static_cast<int>(cr->calls++ & 1);
  const LayerWs w = layer_ws(sh);
  const LayerBufs bufs = layer_bufs(ws, w);
  float* logits = at<float>(ws, w.logits[b]);
  uint16_t* x = at<uint16_t>(ws, w.x[b]);
  uint16_t* out = at<uint16_t>(ws, w.out[b]);
  const int32_t P = sh->P, N = sh->N, H = sh->H;
  const size_t row_bytes = static_cast<size_t>(H) * 2;
  const int32_t T = (minibatch_tokens <= 0 || minibatch_tokens >= N) ? N : minibatch_tokens;
  const int32_t S = N == 0 ? 0 : (N + T - 1) / T;
  auto copy_rows = [&](void* dst, const void* src, int32_t t0, int32_t tm, cudaMemcpyKind kind,
                       cudaStream_t cs) -> cudaError_t {
    for (int32_t r = 0; r < P; ++r) {
      const size_t off = (static_cast<size_t>(r) * N + t0) * row_bytes;
      cudaError_t ee = cudaMemcpyAsync(static_cast<char*>(dst) + off,
                                       static_cast<const char*>(src) + off, tm * row_bytes, kind, cs);
      if (ee != cudaSuccess) return ee;
    }
    return cudaSuccess;
  };
  // the input copies of parity b are free once call i-2 has read them
  if ((e = cudaStreamWaitEvent(cr->h2d, cr->in_free[b], 0)) != cudaSuccess) return e;
  const size_t tokens = static_cast<size_t>(P) * N;
  if ((e = cudaMemcpyAsync(logits, logits_host, tokens * sh->E * 4, cudaMemcpyHostToDevice,
                           cr->h2d)) != cudaSuccess)
    return e;
  if ((e = cudaEventRecord(cr->lg, cr->h2d)) != cudaSuccess) return e;
  if (S > 0) {
    if ((e = copy_rows(x, x_host, 0, T < N ? T : N, cudaMemcpyHostToDevice, cr->h2d)) != cudaSuccess)
      return e;
    if ((e = cudaEventRecord(cr->ex[0], cr->h2d)) != cudaSuccess) return e;
  }
  if ((e = cudaStreamWaitEvent(s, cr->lg, 0)) != cudaSuccess) return e;
  // the device output copy of parity b has been copied out by call i-2
  if ((e = cudaStreamWaitEvent(s, cr->out_free[b], 0)) != cudaSuccess) return e;
  const ZeroSpec z = call_zeroes(bufs, sh);
  if ((e = launch_route_topk(logits, bufs.ids, bufs.gates, static_cast<int64_t>(tokens), sh->E,
                             sh->k, s, &z)) != cudaSuccess)
    return e;
  for (int32_t i = 0; i < S; ++i) {
    const int32_t t0 = i * T, tm = (N - t0) < T ? (N - t0) : T;
    if (i + 1 < S) {  // prefetch the next slice's rows
      const int32_t t1 = t0 + T, tm1 = (N - t1) < T ? (N - t1) : T;
      if ((e = copy_rows(x, x_host, t1, tm1, cudaMemcpyHostToDevice, cr->h2d)) != cudaSuccess)
        return e;
      if ((e = cudaEventRecord(cr->ex[(i + 1) % kRing], cr->h2d)) != cudaSuccess) return e;
    }
    if ((e = cudaStreamWaitEvent(s, cr->ex[i % kRing], 0)) != cudaSuccess) return e;
    if ((e = run_slice(bufs, x, W1, W3, W2, out, Slice{t0, tm}, sh, dev_status, s, nullptr,
                       i == 0)) != cudaSuccess)
      return e;
    if ((e = cudaEventRecord(cr->ed[i % kRing], s)) != cudaSuccess) return e;
    if ((e = cudaStreamWaitEvent(cr->d2h, cr->ed[i % kRing], 0)) != cudaSuccess) return e;
    if ((e = copy_rows(out_host, out, t0, tm, cudaMemcpyDeviceToHost, cr->d2h)) != cudaSuccess)
      return e;
  }
  // routing and every slice's dispatch have read this call's input copies
  if ((e = cudaEventRecord(cr->in_free[b], s)) != cudaSuccess) return e;
  if ((e = cudaEventRecord(cr->out_free[b], cr->d2h)) != cudaSuccess) return e;
  if (out_ready) {
    // the caller waits on out_ready for out_host; `s` goes on computing
    if ((e = cudaEventRecord(out_ready, cr->d2h)) != cudaSuccess) return e;
  } else {
    // `s` completes only after the last copy out
    if ((e = cudaEventRecord(cr->fin, cr->d2h)) != cudaSuccess) return e;
    if ((e = cudaStreamWaitEvent(s, cr->fin, 0)) != cudaSuccess) return e;
  }
  // ... and after every copy in
  if ((e = cudaEventRecord(cr->fin, cr->h2d)) != cudaSuccess) return e;
  return cudaStreamWaitEvent(s, cr->fin, 0);
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
  if (!aligned16(ids) || !aligned16(phi) || !aligned16(route_row) || !aligned32(ws))
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
  if (!aligned16(xg) || !aligned16(W1) || !aligned16(W3) || !aligned16(W2) || !aligned32(h) ||
      !aligned32(y))
    return MOE_INVALID_ARG;
  return from_cuda(launch_expert_ffn(xg, W1, W3, W2, offsets, counts, h, y, *shape,
                                     rows_max_of(shape), dev_status,
                                     static_cast<cudaStream_t>(stream), nullptr));
}

moe_status_t moe_expert_ffn_gather(const uint16_t* x, const int32_t* phi, const uint16_t* W1,
                                   const uint16_t* W3, const uint16_t* W2, const int32_t* offsets,
                                   const int32_t* counts, uint16_t* h, float* y,
                                   int32_t* dev_status, const moe_shape_t* shape, void* stream) {
  moe_status_t st = check_ffn_shape(shape);
  if (st != MOE_OK) return st;
  if (!phi || !W1 || !W3 || !W2 || !offsets || !h || !y || !dev_status ||
      (shape->N > 0 && !x))
    return MOE_INVALID_ARG;
  if (!aligned16(x) || !aligned16(phi) || !aligned16(W1) || !aligned16(W3) || !aligned16(W2) ||
      !aligned32(h) || !aligned32(y))
    return MOE_INVALID_ARG;
  return from_cuda(launch_expert_ffn_gather(x, phi, W1, W3, W2, offsets, counts, h, y, *shape,
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
      !aligned16(out) || !aligned32(ws))
    return MOE_INVALID_ARG;
  if (minibatch_tokens < 0) return MOE_INVALID_ARG;
  if (ws_bytes < layer_ws(shape).total) return MOE_WORKSPACE_TOO_SMALL;
  return layer_body(logits, x, W1, W3, W2, out, minibatch_tokens, ws, dev_status, shape,
                    static_cast<cudaStream_t>(stream), stage_events);
}

size_t moe_train_workspace_bytes(const moe_shape_t* shape) {
  if (check_bwd_shape(shape) != MOE_OK) return 0;
  return layer_ws(shape).total_train;
}

moe_status_t moe_expert_ffn_train(const uint16_t* xg, const uint16_t* W1, const uint16_t* W3,
                                  const uint16_t* W2, const int32_t* offsets,
                                  const int32_t* counts, uint16_t* h, uint16_t* ab, float* y,
                                  int32_t* dev_status, const moe_shape_t* shape, void* stream) {
  moe_status_t st = check_bwd_shape(shape);
  if (st != MOE_OK) return st;
  if (!xg || !W1 || !W3 || !W2 || !offsets || !h || !ab || !y || !dev_status)
    return MOE_INVALID_ARG;
  if (!aligned16(xg) || !aligned16(W1) || !aligned16(W3) || !aligned16(W2) || !aligned32(h) ||
      !aligned32(ab) || !aligned32(y))
    return MOE_INVALID_ARG;
  return from_cuda(launch_expert_ffn(xg, W1, W3, W2, offsets, counts, h, y, *shape,
                                     rows_max_of(shape), dev_status,
                                     static_cast<cudaStream_t>(stream), nullptr, ab));
}

moe_status_t moe_layer_forward_train(const float* logits, const uint16_t* x, const uint16_t* W1,
                                     const uint16_t* W3, const uint16_t* W2, uint16_t* out,
                                     void* ws, size_t ws_bytes, int32_t* dev_status,
                                     const moe_shape_t* shape, void* stream,
                                     void* const* stage_events) {
  moe_status_t st = check_bwd_shape(shape);
  if (st != MOE_OK) return st;
  if (!W1 || !W3 || !W2 || !ws || !dev_status || (shape->N > 0 && (!logits || !x || !out)))
    return MOE_INVALID_ARG;
  if (!aligned16(logits) || !aligned16(x) || !aligned16(W1) || !aligned16(W3) || !aligned16(W2) ||
      !aligned16(out) || !aligned32(ws))
    return MOE_INVALID_ARG;
  if (ws_bytes < layer_ws(shape).total_train) return MOE_WORKSPACE_TOO_SMALL;
  return layer_body(logits, x, W1, W3, W2, out, 0, ws, dev_status, shape,
                    static_cast<cudaStream_t>(stream), stage_events, true);
}

moe_status_t moe_reverse_combine(const uint16_t* dout, const int32_t* phi, const int32_t* offsets,
                                 const int32_t* route_row, const float* gates, uint16_t* dys,
                                 float* gate_row, int32_t* dev_status, const moe_shape_t* shape,
                                 void* stream) {
  moe_status_t st = check_shape(shape);
  if (st != MOE_OK) return st;
  if (shape->H < 8 || shape->H % 8 != 0) return MOE_UNSUPPORTED_SHAPE;
  if (!phi || !offsets || !dys || !gate_row || !dev_status ||
      (shape->N > 0 && (!dout || !route_row || !gates)))
    return MOE_INVALID_ARG;
  if (!aligned16(dout) || !aligned16(phi) || !aligned16(dys)) return MOE_INVALID_ARG;
  return from_cuda(launch_reverse_combine(dout, phi, offsets, route_row, gates, dys, gate_row,
                                          *shape, rows_max_of(shape), dev_status,
                                          static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_expert_ffn_dgrad(const uint16_t* dys, const float* gate_row, const uint16_t* ab,
                                  const uint16_t* h, const uint16_t* W1, const uint16_t* W3,
                                  const uint16_t* W2, const int32_t* offsets,
                                  const int32_t* counts, uint16_t* dab, uint16_t* hg,
                                  float* dgate_part, float* dxg, int32_t* dev_status,
                                  const moe_shape_t* shape, void* stream) {
  moe_status_t st = check_bwd_shape(shape);
  if (st != MOE_OK) return st;
  if (!dys || !gate_row || !ab || !h || !W1 || !W3 || !W2 || !offsets || !dab || !hg ||
      !dgate_part || !dxg || !dev_status)
    return MOE_INVALID_ARG;
  if (!aligned16(dys) || !aligned16(ab) || !aligned16(h) || !aligned16(W1) || !aligned16(W3) ||
      !aligned16(W2) || !aligned16(dab) || !aligned16(hg) || !aligned16(dxg))
    return MOE_INVALID_ARG;
  return from_cuda(launch_expert_ffn_dgrad(dys, gate_row, ab, h, W1, W3, W2, offsets, counts, dab,
                                           hg, dgate_part, dxg, *shape, rows_max_of(shape),
                                           dev_status, static_cast<cudaStream_t>(stream), nullptr));
}

moe_status_t moe_reverse_dispatch(const float* dxg, const int32_t* route_row, uint16_t* dx,
                                  int32_t* dev_status, const moe_shape_t* shape, void* stream) {
  moe_status_t st = check_shape(shape);
  if (st != MOE_OK) return st;
  if (shape->H < 4 || shape->H % 4 != 0) return MOE_UNSUPPORTED_SHAPE;
  if (!dev_status || (shape->N > 0 && (!dxg || !route_row || !dx))) return MOE_INVALID_ARG;
  if (!aligned16(dxg) || !aligned16(dx)) return MOE_INVALID_ARG;
  return from_cuda(launch_reverse_dispatch(dxg, route_row, dx, *shape, rows_max_of(shape),
                                           dev_status, static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_router_backward(const float* dgate_part, const int32_t* route_row,
                                 const int32_t* ids, const float* gates, float* dlogits,
                                 int32_t* dev_status, const moe_shape_t* shape, void* stream) {
  moe_status_t st = check_shape(shape);
  if (st != MOE_OK) return st;
  if (shape->I < 128 || shape->I % 128 != 0) return MOE_UNSUPPORTED_SHAPE;
  if (!dev_status || (shape->N > 0 && (!dgate_part || !route_row || !ids || !gates || !dlogits)))
    return MOE_INVALID_ARG;
  return from_cuda(launch_router_backward(dgate_part, shape->I / 128, route_row, ids, gates, dlogits,
                                          static_cast<int64_t>(shape->P) * shape->N, shape->E,
                                          shape->k, rows_max_of(shape), dev_status,
                                          static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_expert_ffn_wgrad(const uint16_t* xg, const uint16_t* dys, const uint16_t* dab,
                                  const uint16_t* hg, const int32_t* offsets,
                                  const int32_t* counts, float* dW1, float* dW3, float* dW2,
                                  int32_t* dev_status, const moe_shape_t* shape, void* stream) {
  moe_status_t st = check_bwd_shape(shape);
  if (st != MOE_OK) return st;
  if (!xg || !dys || !dab || !hg || !offsets || !dW1 || !dW3 || !dW2 || !dev_status)
    return MOE_INVALID_ARG;
  if (!aligned16(xg) || !aligned16(dys) || !aligned16(dab) || !aligned16(hg) || !aligned32(dW1) ||
      !aligned32(dW3) || !aligned32(dW2))
    return MOE_INVALID_ARG;
  return from_cuda(launch_expert_ffn_wgrad(xg, dys, dab, hg, offsets, counts, dW1, dW3, dW2, *shape,
                                           rows_max_of(shape), dev_status,
                                           static_cast<cudaStream_t>(stream), nullptr));
}

moe_status_t moe_layer_backward(const uint16_t* dout, const uint16_t* W1, const uint16_t* W3,
                                const uint16_t* W2, uint16_t* dx, float* dlogits, float* dW1,
                                float* dW3, float* dW2, void* ws, size_t ws_bytes,
                                int32_t* dev_status, const moe_shape_t* shape, void* stream,
                                void* const* stage_events) {
  moe_status_t st = check_bwd_shape(shape);
  if (st != MOE_OK) return st;
  if (!W1 || !W3 || !W2 || !dW1 || !dW3 || !dW2 || !ws || !dev_status ||
      (shape->N > 0 && (!dout || !dx || !dlogits)))
    return MOE_INVALID_ARG;
  if (!aligned16(dout) || !aligned16(W1) || !aligned16(W3) || !aligned16(W2) || !aligned16(dx) ||
      !aligned32(dW1) || !aligned32(dW3) || !aligned32(dW2) || !aligned32(ws))
    return MOE_INVALID_ARG;
  if (ws_bytes < layer_ws(shape).total_train) return MOE_WORKSPACE_TOO_SMALL;
  return from_cuda(backward_body(dout, W1, W3, W2, dx, dlogits, dW1, dW3, dW2, ws, dev_status,
                                 shape, static_cast<cudaStream_t>(stream), stage_events));
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
  if (!aligned16(W1) || !aligned16(W3) || !aligned16(W2) || !aligned32(ws))
    return MOE_INVALID_ARG;
  if (minibatch_tokens < 0) return MOE_INVALID_ARG;
  const LayerWs w = layer_ws(shape);
  if (ws_bytes < w.total_host) return MOE_WORKSPACE_TOO_SMALL;
  return from_cuda(layer_host_pipeline(logits_host, x_host, W1, W3, W2, out_host, minibatch_tokens,
                                       ws, dev_status, shape, static_cast<cudaStream_t>(stream),
                                       nullptr));
}

moe_status_t moe_layer_forward_host_async(const float* logits_host, const uint16_t* x_host,
                                          const uint16_t* W1, const uint16_t* W3,
                                          const uint16_t* W2, uint16_t* out_host,
                                          int32_t minibatch_tokens, void* ws, size_t ws_bytes,
                                          int32_t* dev_status, const moe_shape_t* shape,
                                          void* stream, void* out_ready) {
  moe_status_t st = check_ffn_shape(shape);
  if (st != MOE_OK) return st;
  if (!out_ready || !W1 || !W3 || !W2 || !ws || !dev_status ||
      (shape->N > 0 && (!logits_host || !x_host || !out_host)))
    return MOE_INVALID_ARG;
  if (!aligned16(W1) || !aligned16(W3) || !aligned16(W2) || !aligned32(ws))
    return MOE_INVALID_ARG;
  if (minibatch_tokens < 0) return MOE_INVALID_ARG;
  if (ws_bytes < layer_ws(shape).total_host) return MOE_WORKSPACE_TOO_SMALL;
  return from_cuda(layer_host_pipeline(logits_host, x_host, W1, W3, W2, out_host, minibatch_tokens,
                                       ws, dev_status, shape, static_cast<cudaStream_t>(stream),
                                       static_cast<cudaEvent_t>(out_ready)));
}

moe_status_t moe_mx_quantize_rows(const uint16_t* src, int64_t n_rows, int32_t K, uint8_t* q,
                                  uint8_t* scale, void* stream) {
  if (n_rows < 0 || K < 32 || K % 32 != 0) return MOE_INVALID_ARG;
  if (n_rows > 0 && (!src || !q || !scale)) return MOE_INVALID_ARG;
  if (!aligned16(src) || !aligned16(q)) return MOE_INVALID_ARG;
  return from_cuda(launch_mx_quantize_rows(src, n_rows, K, q, scale,
                                           static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_dispatch_mxfp8(const uint16_t* x, const int32_t* phi, const int32_t* offsets,
                                uint8_t* xq, uint8_t* xs, int32_t* dev_status,
                                const moe_shape_t* shape, void* stream) {
  moe_status_t st = check_shape(shape);
  if (st != MOE_OK) return st;
  if (shape->H < 32 || shape->H % 32 != 0) return MOE_UNSUPPORTED_SHAPE;
  if (!phi || !offsets || !xq || !xs || !dev_status || (shape->N > 0 && !x)) return MOE_INVALID_ARG;
  if (!aligned16(x) || !aligned16(phi) || !aligned16(xq)) return MOE_INVALID_ARG;
  return from_cuda(launch_dispatch_mxfp8(x, phi, offsets, xq, xs, *shape, rows_max_of(shape),
                                         dev_status, static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_dispatch_mxfp8_tiled(const uint16_t* x, const int32_t* phi,
                                      const int32_t* offsets, uint8_t* xq, uint8_t* xs,
                                      int32_t* dev_status, const moe_shape_t* shape,
                                      void* stream) {
  moe_status_t st = check_shape(shape);
  if (st != MOE_OK) return st;
  if (shape->H < 128 || shape->H % 128 != 0) return MOE_UNSUPPORTED_SHAPE;
  if (!phi || !offsets || !xq || !xs || !dev_status || (shape->N > 0 && !x)) return MOE_INVALID_ARG;
  if (!aligned16(x) || !aligned16(phi) || !aligned16(xq)) return MOE_INVALID_ARG;
  return from_cuda(launch_dispatch_mxfp8(x, phi, offsets, xq, xs, *shape, rows_max_of(shape),
                                         dev_status, static_cast<cudaStream_t>(stream),
                                         /*tiled=*/true));
}

moe_status_t moe_mx_quantize_weights(const uint16_t* W, int32_t E, int32_t K, int32_t N,
                                     uint8_t* q, uint8_t* scale, void* stream) {
  if (E < 0 || K < 128 || K % 128 != 0 || N < 128 || N % 128 != 0) return MOE_INVALID_ARG;
  if (static_cast<int64_t>(E) * K * N >= (int64_t{1} << 40)) return MOE_UNSUPPORTED_SHAPE;
  if (E > 0 && (!W || !q || !scale)) return MOE_INVALID_ARG;
  if (!aligned16(W) || !aligned16(q)) return MOE_INVALID_ARG;
  return from_cuda(launch_mx_quantize_weights(W, E, K, N, q, scale,
                                              static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_expert_ffn_mxfp8(const uint8_t* xq, const uint8_t* xs, const uint8_t* W1q,
                                  const uint8_t* W1s, const uint8_t* W3q, const uint8_t* W3s,
                                  const uint8_t* W2q, const uint8_t* W2s, const int32_t* offsets,
                                  const int32_t* counts, uint8_t* hq, uint8_t* hs, float* y,
                                  int32_t* dev_status, const moe_shape_t* shape, void* stream) {
  moe_status_t st = check_mx_shape(shape);
  if (st != MOE_OK) return st;
  if (!xq || !xs || !W1q || !W1s || !W3q || !W3s || !W2q || !W2s || !offsets || !hq || !hs || !y ||
      !dev_status)
    return MOE_INVALID_ARG;
  if (!aligned16(xq) || !aligned16(xs) || !aligned16(W1q) || !aligned16(W1s) || !aligned16(W3q) ||
      !aligned16(W3s) || !aligned16(W2q) || !aligned16(W2s) || !aligned32(hq) || !aligned16(hs) ||
      !aligned32(y))
    return MOE_INVALID_ARG;
  return from_cuda(launch_expert_ffn_mxfp8(xq, xs, W1q, W1s, W3q, W3s, W2q, W2s, offsets, counts,
                                           hq, hs, y, *shape, rows_max_of(shape), dev_status,
                                           static_cast<cudaStream_t>(stream), nullptr));
}

size_t moe_layer_mxfp8_workspace_bytes(const moe_shape_t* shape) {
  if (check_mx_shape(shape) != MOE_OK) return 0;
  return layer_ws(shape).total_mx;
}

moe_status_t moe_layer_forward_mxfp8(const float* logits, const uint16_t* x, const uint8_t* W1q,
                                     const uint8_t* W1s, const uint8_t* W3q, const uint8_t* W3s,
                                     const uint8_t* W2q, const uint8_t* W2s, const uint16_t* Ws1,
                                     const uint16_t* Ws3, const uint16_t* Ws2, uint16_t* out,
                                     void* ws, size_t ws_bytes, int32_t* dev_status,
                                     const moe_shape_t* shape, void* stream,
                                     void* const* stage_events) {
  moe_status_t st = check_mx_shape(shape);
  if (st != MOE_OK) return st;
  if (!W1q || !W1s || !W3q || !W3s || !W2q || !W2s || !ws || !dev_status ||
      (shape->N > 0 && (!logits || !x || !out)))
    return MOE_INVALID_ARG;
  const bool shared = Ws1 || Ws3 || Ws2;
  if (shared && !(Ws1 && Ws3 && Ws2)) return MOE_INVALID_ARG;  // all three or none
  if (!aligned16(logits) || !aligned16(x) || !aligned16(W1q) || !aligned16(W1s) ||
      !aligned16(W3q) || !aligned16(W3s) || !aligned16(W2q) || !aligned16(W2s) ||
      !aligned16(Ws1) || !aligned16(Ws3) || !aligned16(Ws2) || !aligned16(out) || !aligned32(ws))
    return MOE_INVALID_ARG;
  const LayerWs w = layer_ws(shape);
  if (ws_bytes < (shared ? w.total_mx : w.total)) return MOE_WORKSPACE_TOO_SMALL;
  return from_cuda(layer_body_mx(logits, x, W1q, W1s, W3q, W3s, W2q, W2s, Ws1, Ws3, Ws2, out, ws,
                                 dev_status, shape, static_cast<cudaStream_t>(stream),
                                 stage_events));
}

int64_t moe_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

moe_status_t moe_selftest_bounded_wait(int32_t* dev_status, int64_t timeout_ns, void* stream) {
  if (!dev_status || timeout_ns <= 0) return MOE_INVALID_ARG;
  return from_cuda(launch_selftest_wait(dev_status, timeout_ns, static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_selftest_schedule_barrier(const int32_t* ids, int32_t* phi, int32_t* offsets,
                                           int32_t* counts, int32_t* route_row, void* ws,
                                           size_t ws_bytes, int32_t* dev_status,
                                           const moe_shape_t* shape, int64_t timeout_ns,
                                           void* stream) {
  moe_status_t st = check_shape(shape);
  if (st != MOE_OK) return st;
  if (!phi || !offsets || !counts || !dev_status || !ws || timeout_ns <= 0) return MOE_INVALID_ARG;
  if (shape->N < 1 || !ids || !route_row) return MOE_INVALID_ARG;
  if (!aligned16(ids) || !aligned16(phi) || !aligned16(route_row) || !aligned32(ws))
    return MOE_INVALID_ARG;
  if (ws_bytes < schedule_ws_bytes(shape->P, shape->N, shape->k, shape->E))
    return MOE_WORKSPACE_TOO_SMALL;
  const cudaError_t e = launch_schedule_barrier_selftest(
      ids, *shape, phi, offsets, counts, route_row, static_cast<int32_t*>(ws), dev_status,
      timeout_ns, static_cast<cudaStream_t>(stream));
  if (e == cudaErrorInvalidConfiguration) return MOE_UNSUPPORTED_SHAPE;
  return from_cuda(e);
}

}  // extern "C"
