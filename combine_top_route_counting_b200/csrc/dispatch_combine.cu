// Steps 3a and 4: pull dispatch and fixed-order push combine, and their
// backward twins, which read the same table: pull-reverse-combine and
// push-reverse-dispatch ("Mixture-of-Kittens: A MoE Megakernel for GB300
// NVL72", section 2: forward = pull-dispatch / push-combine, backward =
// pull-reverse-combine / push-reverse-dispatch, one Phi for all four).
//
// Dispatch ("Beyond Peak TFLOPs", section 2.A; "Mixture-of-Kittens: A MoE
// Megakernel for GB300 NVL72", section 2): the destination reads each row's
// source token (src_rank, src_idx) from the two-column table Phi and lands it
// in a contiguous per-expert buffer. On one GPU this is an HBM-to-HBM row
// gather: one warp per row, 16-byte vector loads and stores, four in flight
// per lane; padding rows are written as zeros.
//
// Reverse combine: the dispatch gather applied to the upstream gradient,
// dys[row] = dout[src_rank * N + src_idx], plus the gate of the row's route,
// gate_row[row] = gates[t, j] for the slot j with route_row[t, j] == row (a
// warp ballot over the token's k slots); padding rows get zeros.
//
// Reverse dispatch: dx[t] = bf16_rne(sum_j dxg[route_row[t, j]]) in ascending
// slot order from 0, the combine below with unit weights.
//
// Combine ("Scan once, scatter once", opening: the floating-point order is
// fixed so identical inputs give bitwise-identical outputs): out[t] =
// bf16_rne(acc), acc = 0.0f; acc = fmaf(g[t,j], y[route_row[t,j]], acc) for
// j = 0..k-1. Each output element belongs to one thread and is accumulated in
// ascending slot order, so the result does not depend on scheduling. One
// block per token; each thread issues the k row loads of its 4 columns before
// the k fused multiply-adds.
#include <cuda_bf16.h>

#include "internal.cuh"

namespace moe {
namespace {

constexpr int kMaxK = 16;

// GATE (reverse combine): also gate_row[row] from route_row and gates.
template <bool GATE>
__global__ void __launch_bounds__(256) dispatch_kernel(const uint4* __restrict__ x,
                                                       const int2* __restrict__ phi,
                                                       const int32_t* __restrict__ offsets,
                                                       uint4* __restrict__ xg, int P, int N, int E,
                                                       int H, int64_t rows_max,
                                                       int32_t* dev_status,
                                                       const int32_t* __restrict__ route_row,
                                                       const float* __restrict__ gates,
                                                       float* __restrict__ gate_row, int k) {
  const int rows = __ldg(offsets + E);
  if (rows < 0 || rows > rows_max) {
    if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(dev_status, MOE_DEV_BAD_SCHEDULE);
    return;
  }
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * 8;
  const int nv = H / 8;  // 16-byte vectors per row
  int bad = 0;
  for (int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5); row < rows;
       row += nwarps) {
    const int2 src = __ldg(phi + row);
    uint4* dst = xg + row * nv;
    const bool ok = src.x >= 0 && src.x < P && src.y >= 0 && src.y < N;
    if (!ok) {
      if (src.x >= 0 || src.y != -1) bad = 1;  // (-1,-1) is padding; anything else is corrupt
      const uint4 z = make_uint4(0, 0, 0, 0);
      for (int v = lane; v < nv; v += 32) dst[v] = z;
      if (GATE && lane == 0) gate_row[row] = 0.0f;
      continue;
    }
    const int64_t tok = static_cast<int64_t>(src.x) * N + src.y;
    if (GATE) {
      const int rr = lane < k ? __ldg(route_row + tok * k + lane) : -1;
      const unsigned hit = __ballot_sync(0xFFFFFFFFu, rr == row);
      if (hit == 0u) bad = 1;  // Phi and route_row disagree
      if (lane == 0) gate_row[row] = hit ? __ldg(gates + tok * k + (__ffs(hit) - 1)) : 0.0f;
    }
    const uint4* s = x + tok * nv;
    int v = lane;
    for (; v + 96 < nv; v += 128) {
      const uint4 a = __ldg(s + v), b = __ldg(s + v + 32), c = __ldg(s + v + 64),
                  d = __ldg(s + v + 96);
      dst[v] = a;
      dst[v + 32] = b;
      dst[v + 64] = c;
      dst[v + 96] = d;
    }
    for (; v < nv; v += 32) dst[v] = __ldg(s + v);
  }
  if (bad) atomicOr(dev_status, MOE_DEV_BAD_SCHEDULE);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat16 a = __float2bfloat16_rn(lo);
  const __nv_bfloat16 b = __float2bfloat16_rn(hi);
  return static_cast<uint32_t>(__bfloat16_as_ushort(a)) |
         (static_cast<uint32_t>(__bfloat16_as_ushort(b)) << 16);
}

// K > 0: compile-time k; K == 0: runtime k (<= kMaxK). gates == null: unit
// weights (fmaf(1, v, acc) is the rounded sum acc + v). SHARED: the sum
// starts from the shared expert's output row shared[t] instead of 0 (the
// shared expert as a slot before slot 0 with gate 1).
template <int K, bool SHARED = false>
__global__ void __launch_bounds__(256) combine_kernel(const float4* __restrict__ y,
                                                      const int32_t* __restrict__ route_row,
                                                      const float* __restrict__ gates,
                                                      uint2* __restrict__ out, int N, int k, int H,
                                                      int t0, int Tm, int64_t rows_max,
                                                      int32_t* dev_status,
                                                      const float4* __restrict__ shared) {
  constexpr int KM = K > 0 ? K : kMaxK;
  const int kk = K > 0 ? K : k;
  const int64_t b = blockIdx.x;  // token of the slice, peer-major
  const int r = static_cast<int>(b / Tm), i = static_cast<int>(b - static_cast<int64_t>(r) * Tm);
  const int64_t t = static_cast<int64_t>(r) * N + t0 + i;
  const int nv = H / 4;
  int64_t rows[KM];
  float g[KM];
  int bad = 0;
#pragma unroll
  for (int j = 0; j < KM; ++j) {
    rows[j] = -1;
    g[j] = 0.0f;
    if (j < kk) {
      const int rr = __ldg(route_row + t * k + j);
      g[j] = gates ? __ldg(gates + t * k + j) : 1.0f;
      if (rr >= 0 && rr < rows_max)
        rows[j] = rr;
      else
        bad = 1;
    }
  }
  if (bad && threadIdx.x == 0) atomicOr(dev_status, MOE_DEV_BAD_SCHEDULE);
  for (int v = threadIdx.x; v < nv; v += 256) {
    float4 val[KM];
#pragma unroll
    for (int j = 0; j < KM; ++j)
      if (j < kk && rows[j] >= 0) val[j] = __ldg(y + rows[j] * nv + v);
    float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    if (SHARED) acc = __ldg(shared + t * nv + v);
#pragma unroll
    for (int j = 0; j < KM; ++j) {
      if (j < kk && rows[j] >= 0) {
        acc.x = __fmaf_rn(g[j], val[j].x, acc.x);
        acc.y = __fmaf_rn(g[j], val[j].y, acc.y);
        acc.z = __fmaf_rn(g[j], val[j].z, acc.z);
        acc.w = __fmaf_rn(g[j], val[j].w, acc.w);
      }
    }
    out[t * nv + v] = make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
  }
}

}  // namespace

cudaError_t launch_dispatch(const uint16_t* x, const int32_t* phi, const int32_t* offsets,
                            uint16_t* xg, const moe_shape_t& sh, int64_t rows_max,
                            int32_t* dev_status, cudaStream_t s) {
  if (rows_max <= 0) return cudaSuccess;
  const int64_t want = (rows_max + 7) / 8;
  const int64_t cap = static_cast<int64_t>(device_sm_count()) * 8;
  const int blocks = static_cast<int>(want < cap ? want : cap);
  dispatch_kernel<false><<<blocks, 256, 0, s>>>(reinterpret_cast<const uint4*>(x),
                                                reinterpret_cast<const int2*>(phi), offsets,
                                                reinterpret_cast<uint4*>(xg), sh.P, sh.N, sh.E,
                                                sh.H, rows_max, dev_status, nullptr, nullptr,
                                                nullptr, sh.k);
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_reverse_combine(const uint16_t* dout, const int32_t* phi,
                                   const int32_t* offsets, const int32_t* route_row,
                                   const float* gates, uint16_t* dys, float* gate_row,
                                   const moe_shape_t& sh, int64_t rows_max, int32_t* dev_status,
                                   cudaStream_t s) {
  if (rows_max <= 0) return cudaSuccess;
  const int64_t want = (rows_max + 7) / 8;
  const int64_t cap = static_cast<int64_t>(device_sm_count()) * 8;
  const int blocks = static_cast<int>(want < cap ? want : cap);
  dispatch_kernel<true><<<blocks, 256, 0, s>>>(reinterpret_cast<const uint4*>(dout),
                                               reinterpret_cast<const int2*>(phi), offsets,
                                               reinterpret_cast<uint4*>(dys), sh.P, sh.N, sh.E,
                                               sh.H, rows_max, dev_status, route_row, gates,
                                               gate_row, sh.k);
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_combine(const float* y, const int32_t* route_row, const float* gates,
                           uint16_t* out, const moe_shape_t& sh, Slice sl, int64_t rows_max,
                           int32_t* dev_status, cudaStream_t s, const float* shared) {
  const int64_t tokens = static_cast<int64_t>(sh.P) * sl.Tm;
  if (tokens == 0) return cudaSuccess;
  const float4* y4 = reinterpret_cast<const float4*>(y);
  const float4* s4 = reinterpret_cast<const float4*>(shared);
  uint2* o2 = reinterpret_cast<uint2*>(out);
  const unsigned grid = static_cast<unsigned>(tokens);
#define MOE_COMBINE(KV, SH)                                                                     \
  combine_kernel<KV, SH><<<grid, 256, 0, s>>>(y4, route_row, gates, o2, sh.N, sh.k, sh.H, sl.t0, \
                                              sl.Tm, rows_max, dev_status, s4)
  if (shared) {
    switch (sh.k) {
      case 8: MOE_COMBINE(8, true); break;
      default: MOE_COMBINE(0, true); break;
    }
  } else {
    switch (sh.k) {
      case 1: MOE_COMBINE(1, false); break;
      case 2: MOE_COMBINE(2, false); break;
      case 4: MOE_COMBINE(4, false); break;
      case 8: MOE_COMBINE(8, false); break;
      default: MOE_COMBINE(0, false); break;
    }
  }
#undef MOE_COMBINE
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_reverse_dispatch(const float* dxg, const int32_t* route_row, uint16_t* dx,
                                    const moe_shape_t& sh, int64_t rows_max, int32_t* dev_status,
                                    cudaStream_t s) {
  return launch_combine(dxg, route_row, nullptr, dx, sh, Slice{0, sh.N}, rows_max, dev_status, s);
}

}  // namespace moe
