// Step 1: top-k routing and gates.
//
// "Mixture-of-Kittens: A MoE Megakernel for GB300 NVL72", section 2: the
// schedule is built from the routing tensor (each token's k experts). For
// every token the k largest logits are taken in descending order, ties to the
// lower expert id; the gates are the softmax over those k logits.
//
// One warp per token. Lane `lane` holds logits lane, lane+32, ... (each
// register column is one coalesced 128-byte load). Each of the k rounds is a
// lane-local best followed by a butterfly argmax over the warp under the
// total order (value descending, id ascending); the owner lane marks the
// winner as taken. HBM-bound: the logits are read once.
#include <cfloat>
#include <climits>
#include <cmath>

#include "internal.cuh"

namespace moe {
namespace {

constexpr int kMaxK = 16;
constexpr unsigned kFull = 0xFFFFFFFFu;

__device__ __forceinline__ bool better(float v, int id, float bv, int bid) {
  return v > bv || (v == bv && id < bid);
}

template <int VPL>
__global__ void __launch_bounds__(256) route_topk_kernel(const float* __restrict__ logits,
                                                         int32_t* __restrict__ ids,
                                                         float* __restrict__ gates,
                                                         int64_t n_tokens, int E, int k) {
  const int lane = threadIdx.x & 31;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (t >= n_tokens) return;  // whole warp leaves together
  const float* row = logits + t * E;

  float v[VPL];
  uint32_t taken = 0;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int e = i * 32 + lane;
    if (e < E) {
      v[i] = __ldg(row + e);
    } else {
      v[i] = -INFINITY;
      taken |= 1u << i;  // not an expert
    }
  }

  float sel_v[kMaxK];
  int sel_id[kMaxK];
#pragma unroll
  for (int j = 0; j < kMaxK; ++j) {
    sel_v[j] = -INFINITY;
    sel_id[j] = 0;
    if (j < k) {
      float bv = -INFINITY;
      int bid = INT_MAX;
#pragma unroll
      for (int i = 0; i < VPL; ++i) {
        const int e = i * 32 + lane;
        if (!((taken >> i) & 1u) && better(v[i], e, bv, bid)) {
          bv = v[i];
          bid = e;
        }
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const float ov = __shfl_xor_sync(kFull, bv, off);
        const int oid = __shfl_xor_sync(kFull, bid, off);
        if (better(ov, oid, bv, bid)) {
          bv = ov;
          bid = oid;
        }
      }
      if (bid != INT_MAX && (bid & 31) == lane) taken |= 1u << (bid >> 5);
      sel_v[j] = bv;
      sel_id[j] = bid;
    }
  }

  // gates: softmax over the chosen logits, summed in slot order
  const float l0 = sel_v[0];
  float ex[kMaxK];
  float den = 0.0f;
#pragma unroll
  for (int j = 0; j < kMaxK; ++j) {
    ex[j] = 0.0f;
    if (j < k) {
      ex[j] = expf(sel_v[j] - l0);
      den += ex[j];
    }
  }
#pragma unroll
  for (int j = 0; j < kMaxK; ++j) {
    if (j < k && lane == j) {
      ids[t * k + j] = sel_id[j];
      gates[t * k + j] = ex[j] / den;
    }
  }
}

template <int VPL>
cudaError_t launch_vpl(const float* logits, int32_t* ids, float* gates, int64_t n, int E, int k,
                       cudaStream_t s) {
  const int64_t blocks = (n + 7) / 8;
  route_topk_kernel<VPL><<<static_cast<unsigned>(blocks), 256, 0, s>>>(logits, ids, gates, n, E, k);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_route_topk(const float* logits, int32_t* ids, float* gates, int64_t n_tokens,
                              int32_t E, int32_t k, cudaStream_t s) {
  if (n_tokens == 0) return cudaSuccess;
  if (E <= 32) return launch_vpl<1>(logits, ids, gates, n_tokens, E, k, s);
  if (E <= 64) return launch_vpl<2>(logits, ids, gates, n_tokens, E, k, s);
  if (E <= 128) return launch_vpl<4>(logits, ids, gates, n_tokens, E, k, s);
  if (E <= 256) return launch_vpl<8>(logits, ids, gates, n_tokens, E, k, s);
  if (E <= 384) return launch_vpl<12>(logits, ids, gates, n_tokens, E, k, s);
  if (E <= 512) return launch_vpl<16>(logits, ids, gates, n_tokens, E, k, s);
  return launch_vpl<32>(logits, ids, gates, n_tokens, E, k, s);
}

}  // namespace moe
