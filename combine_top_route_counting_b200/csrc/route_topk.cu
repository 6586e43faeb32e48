// Step 1: top-k routing and gates.
//
// "Mixture-of-Kittens: A MoE Megakernel for GB300 NVL72", section 2: the
// schedule is built from the routing tensor (each token's k experts). For
// every token the k largest logits are taken in descending order, ties to the
// lower expert id; the gates are the softmax over those k logits.
//
// One warp per token; lane `lane` holds logits lane, lane+32, ... (each
// register column is one coalesced 128-byte load). Selection avoids k rounds
// of warp-wide argmax:
//   1. tau = the k-th largest of the 32 lane maxima (a warp bitonic sort).
//      These are k actual logits of the token, so tau is at most its k-th
//      largest logit: every chosen expert has a logit >= tau.
//   2. The few logits >= tau (usually a little more than k) are compacted
//      into shared memory; each candidate's rank under the total order
//      (value descending, id ascending) is counted against the others, and
//      ranks 0..k-1 are the slots. Exact: ranks of a total order are unique.
//   3. If more than 32 logits reach tau (heavy ties, -inf logits), the warp
//      falls back to k rounds of butterfly argmax over all its logits.
// HBM-bound: the logits are read once.
#include <cfloat>
#include <climits>
#include <cmath>

#include "internal.cuh"

namespace moe {
namespace {

constexpr int kMaxK = 16;
constexpr int kCand = 32;  // candidate buffer per warp
constexpr unsigned kFull = 0xFFFFFFFFu;

__device__ __forceinline__ bool better(float v, int id, float bv, int bid) {
  return v > bv || (v == bv && id < bid);
}

// Block 0 zeroes the scratch words the call's later kernels expect at zero.
__device__ __forceinline__ void zero_words(const ZeroSpec& z) {
  if (blockIdx.x != 0) return;
  for (int i = threadIdx.x; i < z.na; i += blockDim.x) z.a[i] = 0;
  for (int i = threadIdx.x; i < z.nb; i += blockDim.x) z.b[i] = 0;
}

template <int VPL>
__global__ void __launch_bounds__(256) route_topk_kernel(const float* __restrict__ logits,
                                                         int32_t* __restrict__ ids,
                                                         float* __restrict__ gates,
                                                         int64_t n_tokens, int E, int k,
                                                         ZeroSpec z) {
  zero_words(z);
  __shared__ float s_cv[8][kCand];
  __shared__ int s_ci[8][kCand];
  __shared__ float s_sv[8][kMaxK];
  __shared__ int s_si[8][kMaxK];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * 8 + w;
  if (t >= n_tokens) return;  // whole warp leaves together
  const float* row = logits + t * E;

  float v[VPL];
  float m = -INFINITY;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int e = i * 32 + lane;
    v[i] = (e < E) ? __ldg(row + e) : -INFINITY;
    m = fmaxf(m, v[i]);
  }

  // 1. tau: k-th largest lane maximum (bitonic sort, descending across lanes)
  float x = m;
#pragma unroll
  for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      const float o = __shfl_xor_sync(kFull, x, stride);
      const bool asc = (lane & size) != 0;  // final stage (size 32): descending
      const bool lower = (lane & stride) == 0;
      x = (lower != asc) ? fmaxf(x, o) : fminf(x, o);
    }
  }
  const float tau = __shfl_sync(kFull, x, k - 1);

  // 2. compact the logits >= tau
  int c = 0;
#pragma unroll
  for (int i = 0; i < VPL; ++i) c += (i * 32 + lane < E && v[i] >= tau) ? 1 : 0;
  int incl = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(kFull, incl, o);
    if (lane >= o) incl += y;
  }
  const int total = __shfl_sync(kFull, incl, 31);

  if (total <= kCand) {
    int pos = incl - c;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int e = i * 32 + lane;
      if (e < E && v[i] >= tau) {
        s_cv[w][pos] = v[i];
        s_ci[w][pos] = e;
        ++pos;
      }
    }
    __syncwarp();
    if (lane < total) {
      const float cv = s_cv[w][lane];
      const int ci = s_ci[w][lane];
      int rank = 0;
      for (int j = 0; j < total; ++j) rank += better(s_cv[w][j], s_ci[w][j], cv, ci) ? 1 : 0;
      if (rank < k) {
        s_sv[w][rank] = cv;
        s_si[w][rank] = ci;
      }
    }
  } else {
    // 3. fallback: k rounds of warp argmax over every logit of the token
    uint32_t taken = 0;
#pragma unroll
    for (int i = 0; i < VPL; ++i)
      if (i * 32 + lane >= E) taken |= 1u << i;
    for (int j = 0; j < k; ++j) {
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
      if (lane == 0) {
        s_sv[w][j] = bv;
        s_si[w][j] = bid;
      }
    }
  }
  __syncwarp();

  // gates: softmax over the chosen logits, summed in slot order
  if (lane < k) {
    const float l0 = s_sv[w][0];
    float den = 0.0f;
    for (int j = 0; j < k; ++j) den += expf(s_sv[w][j] - l0);
    ids[t * k + lane] = s_si[w][lane];
    gates[t * k + lane] = expf(s_sv[w][lane] - l0) / den;
  }
}

// Eight lanes per token, four tokens per warp (E a multiple of 4, E <= 512;
// used for E <= 128 or k > 8, the four-lane kernel below for the rest): the
// same selection with a quarter of the shuffle work per token. Lane g of
// a token's group loads float4 chunks g, g+8, g+16, ... of its logit row
// (NV = ceil(E/32) chunks; the group's eight 16-byte loads of one step are
// one 128-byte segment), and keeps its two largest values. tau = the k-th
// largest of the group's 16 kept values under (value desc, position asc) --
// at least k logits of the token are >= tau, so every chosen expert is among
// them. The logits >= tau are compacted to shared memory and ranked exactly
// under (value desc, id asc); more than 32 of them (heavy ties, -inf) fall
// back to k rounds of group-wide argmax. Gates as above, summed in slot order.
template <int NV>
__global__ void __launch_bounds__(256, 2) route_topk_g8_kernel(const float* __restrict__ logits,
                                                            int32_t* __restrict__ ids,
                                                            float* __restrict__ gates,
                                                            int64_t n_tokens, int E, int k,
                                                            ZeroSpec z) {
  zero_words(z);
  // rows padded by one word: the four tokens of a warp read the same
  // candidate index at once, which an unpadded row stride puts in one bank
  __shared__ float s_cv[32][kCand + 1];
  __shared__ int s_ci[32][kCand + 1];
  __shared__ float s_sv[32][kMaxK + 1];
  __shared__ int s_si[32][kMaxK + 1];
  const int lane = threadIdx.x & 31, g = lane & 7, tb = threadIdx.x >> 3;  // token in block
  const int gbase = lane & 24;
  const unsigned gm = 0xFFu << gbase;  // this token's eight lanes
  const int64_t t = static_cast<int64_t>(blockIdx.x) * 32 + tb;
  if (t >= n_tokens) return;  // the whole group leaves together
  const float4* row = reinterpret_cast<const float4*>(logits + t * E);
  const int nv4 = E >> 2;

  float v[NV][4];
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int cidx = g + 8 * i;
    if (cidx < nv4) {
      const float4 q = __ldg(row + cidx);
      v[i][0] = q.x;
      v[i][1] = q.y;
      v[i][2] = q.z;
      v[i][3] = q.w;
    } else {
      v[i][0] = v[i][1] = v[i][2] = v[i][3] = -INFINITY;
    }
  }
  // the lane's two largest values (as a multiset)
  float m1 = -INFINITY, m2 = -INFINITY;
#pragma unroll
  for (int i = 0; i < NV; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      m2 = fmaxf(m2, fminf(m1, v[i][j]));
      m1 = fmaxf(m1, v[i][j]);
    }
  // tau: the value of rank k-1 among the group's 16 kept values, ordered by
  // (value desc, position asc) with position 2h (m1) and 2h+1 (m2) of lane h
  int ra = 0, rb = 0;
#pragma unroll
  for (int h = 0; h < 8; ++h) {
    const float oa = __shfl_sync(gm, m1, gbase | h);
    const float ob = __shfl_sync(gm, m2, gbase | h);
    ra += (oa > m1 || (oa == m1 && h < g)) ? 1 : 0;
    ra += (ob > m1 || (ob == m1 && h < g)) ? 1 : 0;  // 2h+1 < 2g  <=>  h < g
    rb += (oa > m2 || (oa == m2 && h <= g)) ? 1 : 0;  // 2h < 2g+1 <=> h <= g
    rb += (ob > m2 || (ob == m2 && h < g)) ? 1 : 0;
  }
  const unsigned own = __ballot_sync(gm, ra == k - 1 || rb == k - 1) >> gbase;
  const float tau = __shfl_sync(gm, ra == k - 1 ? m1 : m2, gbase | (__ffs(own) - 1));

  // compact the logits >= tau
  int c = 0;
#pragma unroll
  for (int i = 0; i < NV; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) c += (v[i][j] >= tau && (g + 8 * i) < nv4) ? 1 : 0;
  int incl = c;
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) {
    const int y = __shfl_up_sync(gm, incl, o, 8);
    if (g >= o) incl += y;
  }
  const int total = __shfl_sync(gm, incl, gbase | 7);

  if (total <= kCand) {
    int pos = incl - c;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      // most chunks hold no candidate: one test skips them
      if (fmaxf(fmaxf(v[i][0], v[i][1]), fmaxf(v[i][2], v[i][3])) < tau || (g + 8 * i) >= nv4)
        continue;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (v[i][j] >= tau) {
          s_cv[tb][pos] = v[i][j];
          s_ci[tb][pos] = 4 * (g + 8 * i) + j;
          ++pos;
        }
      }
    }
    __syncwarp(gm);
    for (int a = g; a < total; a += 8) {
      const float cv = s_cv[tb][a];
      const int ci = s_ci[tb][a];
      int rank = 0;
      for (int b = 0; b < total; ++b) rank += better(s_cv[tb][b], s_ci[tb][b], cv, ci) ? 1 : 0;
      if (rank < k) {
        s_sv[tb][rank] = cv;
        s_si[tb][rank] = ci;
      }
    }
  } else {
    // fallback: k rounds of group argmax over every logit of the token
    uint64_t taken = 0;
#pragma unroll
    for (int i = 0; i < NV; ++i)
      if (g + 8 * i >= nv4) taken |= 0xFull << (4 * i);
    for (int r = 0; r < k; ++r) {
      float bv = -INFINITY;
      int bid = INT_MAX;
#pragma unroll
      for (int i = 0; i < NV; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int e = 4 * (g + 8 * i) + j;
          if (!((taken >> (4 * i + j)) & 1ull) && better(v[i][j], e, bv, bid)) {
            bv = v[i][j];
            bid = e;
          }
        }
#pragma unroll
      for (int off = 4; off > 0; off >>= 1) {
        const float ov = __shfl_xor_sync(gm, bv, off, 8);
        const int oid = __shfl_xor_sync(gm, bid, off, 8);
        if (better(ov, oid, bv, bid)) {
          bv = ov;
          bid = oid;
        }
      }
      if (bid != INT_MAX && ((bid >> 2) & 7) == g) {
        const int i = (bid >> 2) >> 3;
        taken |= 1ull << (4 * i + (bid & 3));
      }
      if (g == 0) {
        s_sv[tb][r] = bv;
        s_si[tb][r] = bid;
      }
    }
  }
  __syncwarp(gm);

  // gates: softmax over the chosen logits, summed in slot order (lane g holds
  // slots g and g + 8)
  const float l0 = s_sv[tb][0];
  const float e0 = g < k ? expf(s_sv[tb][g] - l0) : 0.0f;
  const float e1 = g + 8 < k ? expf(s_sv[tb][g + 8] - l0) : 0.0f;
  float den = 0.0f;
  for (int j = 0; j < k; ++j) den += __shfl_sync(gm, j < 8 ? e0 : e1, gbase | (j & 7));
  if (g < k) {
    ids[t * k + g] = s_si[tb][g];
    gates[t * k + g] = e0 / den;
  }
  if (g + 8 < k) {
    ids[t * k + g + 8] = s_si[tb][g + 8];
    gates[t * k + g + 8] = e1 / den;
  }
}

// Four lanes per token, eight tokens per warp (E a multiple of 16, E <= 512,
// k <= 8). Lane g of a token's quad loads float4 chunks g, g+4, g+8, ... of
// the logit row (NC >= E/16 chunks; the quad's four 16-byte loads of one step
// are one 64-byte segment) and keeps each chunk's maximum, plus the four
// largest of them (sorted). tau = the k-th largest value of the quad's 16
// kept chunk maxima (two merge steps of sorted lists across the quad): these
// are actual logits, so at least k logits are >= tau and every chosen expert
// is among them. Only the chunks whose maximum reaches tau are read again
// (from L1); their logits >= tau go to the lane's 16 candidate slots, and
// each candidate's rank under (value desc, id asc) among the quad's
// candidates is counted: ranks 0..k-1 are the slots. More than 16 candidates
// in one lane (heavy ties, -inf logits) send the quad to k rounds of
// quad-wide argmax over all its logits, round r taking the best logit that
// comes after round r-1's in that order. Gates as above, summed in slot order.
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Sorts a bitonic sequence of 8 values into descending order.
__device__ __forceinline__ void bitonic_merge8_desc(float (&c)[8]) {
#pragma unroll
  for (int d = 4; d > 0; d >>= 1)
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if ((i & d) == 0) {
        const float hi = fmaxf(c[i], c[i + d]), lo = fminf(c[i], c[i + d]);
        c[i] = hi;
        c[i + d] = lo;
      }
}

constexpr int kG4Slots = 16;  // candidate slots per lane

template <int NC>
__global__ void __launch_bounds__(256) route_topk_g4_kernel(const float* __restrict__ logits,
                                                            int32_t* __restrict__ ids,
                                                            float* __restrict__ gates,
                                                            int64_t n_tokens, int E, int k,
                                                            ZeroSpec z) {
  static_assert(NC <= 32, "one mask bit per chunk");
  zero_words(z);
  // token rows padded by one word: the eight quads of a warp read the same
  // slot index at once
  __shared__ float s_cv[64][4 * kG4Slots + 1];  // lane g's candidates at [16g, 16g + 16)
  __shared__ int s_ci[64][4 * kG4Slots + 1];
  __shared__ float s_sv[64][9];
  __shared__ int s_si[64][9];
  const int lane = threadIdx.x & 31, g = lane & 3, tb = threadIdx.x >> 2;  // token in block
  const int gbase = lane & 28;
  const unsigned gm = 0xFu << gbase;  // this token's four lanes
  const int64_t t = static_cast<int64_t>(blockIdx.x) * 64 + tb;
  if (t >= n_tokens) return;  // the whole quad leaves together
  const float4* row = reinterpret_cast<const float4*>(logits + t * E);
  const int nc4 = E >> 2;

  // chunk maxima and the lane's four largest of them, descending
  float cm[NC];
  float a[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
  constexpr int kBatch = 12;  // loads in flight per lane
#pragma unroll
  for (int i0 = 0; i0 < NC; i0 += kBatch) {
    float4 q[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int c = g + 4 * (i0 + u);
      if (i0 + u < NC)
        q[u] = c < nc4 ? __ldg(row + c) : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      if (i0 + u < NC) {
        const float v = fmaxf(fmax3(q[u].x, q[u].y, q[u].z), q[u].w);
        cm[i0 + u] = v;
        a[3] = fmaxf(a[3], fminf(a[2], v));
        a[2] = fmaxf(a[2], fminf(a[1], v));
        a[1] = fmaxf(a[1], fminf(a[0], v));
        a[0] = fmaxf(a[0], v);
      }
    }
  }
  // tau: merge with the partner lane (xor 1) into a sorted 8, then keep the
  // top 8 of that and the other pair's sorted 8 (xor 2), sorted
  float c8[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    c8[i] = a[i];
    c8[7 - i] = __shfl_xor_sync(gm, a[i], 1);
  }
  bitonic_merge8_desc(c8);
  float d8[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) d8[7 - i] = __shfl_xor_sync(gm, c8[i], 2);
#pragma unroll
  for (int i = 0; i < 8; ++i) d8[i] = fmaxf(c8[i], d8[i]);
  bitonic_merge8_desc(d8);
  float tau = d8[0];
#pragma unroll
  for (int i = 1; i < 8; ++i)
    if (i == k - 1) tau = d8[i];

  // candidates: the logits >= tau of the chunks whose maximum reaches tau
  unsigned pm = 0;
#pragma unroll
  for (int i = 0; i < NC; ++i)
    if (g + 4 * i < nc4 && cm[i] >= tau) pm |= 1u << i;
  int c = 0;
  while (pm) {
    const int i = __ffs(pm) - 1;
    pm &= pm - 1;
    const int ch = g + 4 * i;
    const float4 q = __ldg(row + ch);
    const float vv[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (vv[j] >= tau) {
        if (c < kG4Slots) {
          s_cv[tb][kG4Slots * g + c] = vv[j];
          s_ci[tb][kG4Slots * g + c] = 4 * ch + j;
        }
        ++c;
      }
    }
  }
  const bool over = (__ballot_sync(gm, c > kG4Slots) & gm) != 0;
  __syncwarp(gm);

  if (!over) {
    // rank every candidate of the quad: lane g takes candidates g, g+4, ...
    // of the quad's list (lane h's slots in order, then lane h+1's)
    int cnt[4], off[5];
    off[0] = 0;
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      cnt[h] = __shfl_sync(gm, c, gbase | h);
      off[h + 1] = off[h] + cnt[h];
    }
    const int total = off[4];
    for (int ai = g; ai < total; ai += 4) {
      const int ha = (ai >= off[1]) + (ai >= off[2]) + (ai >= off[3]);
      const int oa = ha == 0 ? 0 : ha == 1 ? off[1] : ha == 2 ? off[2] : off[3];
      const int sa = kG4Slots * ha + (ai - oa);
      const float cv = s_cv[tb][sa];
      const int ci = s_ci[tb][sa];
      int rank = 0;
#pragma unroll
      for (int h = 0; h < 4; ++h)
        for (int b = 0; b < cnt[h]; ++b)
          rank += better(s_cv[tb][kG4Slots * h + b], s_ci[tb][kG4Slots * h + b], cv, ci) ? 1 : 0;
      if (rank < k) {
        s_sv[tb][rank] = cv;
        s_si[tb][rank] = ci;
      }
    }
  } else {
    float pv = INFINITY;  // round r's pick comes after (pv, pid): none yet
    int pid = -1;
    for (int r = 0; r < k; ++r) {
      float bv = -INFINITY;
      int bid = INT_MAX;
      for (int i = 0; i < NC; ++i) {
        const int ch = g + 4 * i;
        if (ch >= nc4) break;
        const float4 q = __ldg(row + ch);
        const float vv[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int e = 4 * ch + j;
          if (better(pv, pid, vv[j], e) && better(vv[j], e, bv, bid)) {
            bv = vv[j];
            bid = e;
          }
        }
      }
#pragma unroll
      for (int o = 2; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(gm, bv, o, 4);
        const int oid = __shfl_xor_sync(gm, bid, o, 4);
        if (better(ov, oid, bv, bid)) {
          bv = ov;
          bid = oid;
        }
      }
      if (g == 0) {
        s_sv[tb][r] = bv;
        s_si[tb][r] = bid;
      }
      pv = bv;
      pid = bid;
    }
  }
  __syncwarp(gm);

  // gates: softmax over the chosen logits, summed in slot order (lane g holds
  // slots g and g + 4)
  const float l0 = s_sv[tb][0];
  const float e0 = g < k ? expf(s_sv[tb][g] - l0) : 0.0f;
  const float e1 = g + 4 < k ? expf(s_sv[tb][g + 4] - l0) : 0.0f;
  float den = 0.0f;
  for (int j = 0; j < k; ++j) den += __shfl_sync(gm, j < 4 ? e0 : e1, gbase | (j & 3));
  if (g < k) {
    ids[t * k + g] = s_si[tb][g];
    gates[t * k + g] = e0 / den;
  }
  if (g + 4 < k) {
    ids[t * k + g + 4] = s_si[tb][g + 4];
    gates[t * k + g + 4] = e1 / den;
  }
}

template <int NC>
cudaError_t launch_g4(const float* logits, int32_t* ids, float* gates, int64_t n, int E, int k,
                      cudaStream_t s, ZeroSpec z) {
  const int64_t blocks = (n + 63) / 64;
  route_topk_g4_kernel<NC><<<static_cast<unsigned>(blocks), 256, 0, s>>>(logits, ids, gates, n, E,
                                                                         k, z);
  note_launches(1);
  return cudaGetLastError();
}

template <int NV>
cudaError_t launch_g8(const float* logits, int32_t* ids, float* gates, int64_t n, int E, int k,
                      cudaStream_t s, ZeroSpec z) {
  const int64_t blocks = (n + 31) / 32;
  route_topk_g8_kernel<NV><<<static_cast<unsigned>(blocks), 256, 0, s>>>(logits, ids, gates, n, E,
                                                                         k, z);
  note_launches(1);
  return cudaGetLastError();
}

template <int VPL>
cudaError_t launch_vpl(const float* logits, int32_t* ids, float* gates, int64_t n, int E, int k,
                       cudaStream_t s, ZeroSpec z) {
  const int64_t blocks = (n + 7) / 8;
  route_topk_kernel<VPL><<<static_cast<unsigned>(blocks), 256, 0, s>>>(logits, ids, gates, n, E, k,
                                                                       z);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_route_topk(const float* logits, int32_t* ids, float* gates, int64_t n_tokens,
                              int32_t E, int32_t k, cudaStream_t s, const ZeroSpec* zp) {
  const ZeroSpec z = zp ? *zp : ZeroSpec{nullptr, 0, nullptr, 0};
  if (n_tokens == 0) {
    if (z.na > 0 && cudaMemsetAsync(z.a, 0, z.na * sizeof(int), s) != cudaSuccess)
      return cudaGetLastError();
    if (z.nb > 0 && cudaMemsetAsync(z.b, 0, z.nb * sizeof(int), s) != cudaSuccess)
      return cudaGetLastError();
    return cudaSuccess;
  }
  // four lanes per token for the wide rows (at E <= 128 the eight-lane
  // kernel's twice as many blocks fill the device better)
  if (E % 16 == 0 && E > 128 && E <= 512 && k <= 8) {
    if (E <= 192) return launch_g4<12>(logits, ids, gates, n_tokens, E, k, s, z);
    if (E <= 256) return launch_g4<16>(logits, ids, gates, n_tokens, E, k, s, z);
    if (E <= 384) return launch_g4<24>(logits, ids, gates, n_tokens, E, k, s, z);
    return launch_g4<32>(logits, ids, gates, n_tokens, E, k, s, z);
  }
  if (E % 4 == 0 && E <= 512) {
    if (E <= 32) return launch_g8<1>(logits, ids, gates, n_tokens, E, k, s, z);
    if (E <= 64) return launch_g8<2>(logits, ids, gates, n_tokens, E, k, s, z);
    if (E <= 128) return launch_g8<4>(logits, ids, gates, n_tokens, E, k, s, z);
    if (E <= 256) return launch_g8<8>(logits, ids, gates, n_tokens, E, k, s, z);
    if (E <= 384) return launch_g8<12>(logits, ids, gates, n_tokens, E, k, s, z);
    return launch_g8<16>(logits, ids, gates, n_tokens, E, k, s, z);
  }
  if (E <= 32) return launch_vpl<1>(logits, ids, gates, n_tokens, E, k, s, z);
  if (E <= 64) return launch_vpl<2>(logits, ids, gates, n_tokens, E, k, s, z);
  if (E <= 128) return launch_vpl<4>(logits, ids, gates, n_tokens, E, k, s, z);
  if (E <= 256) return launch_vpl<8>(logits, ids, gates, n_tokens, E, k, s, z);
  if (E <= 384) return launch_vpl<12>(logits, ids, gates, n_tokens, E, k, s, z);
  if (E <= 512) return launch_vpl<16>(logits, ids, gates, n_tokens, E, k, s, z);
  return launch_vpl<32>(logits, ids, gates, n_tokens, E, k, s, z);
}

// ---------------------------------------------------------------- backward
// Router gradient ("Mixture-of-Kittens", section 5, SonicMoE gradients: from
// the inner product of the SwiGLU activations and the down-projection
// dgrads). dgate[t, j] = sum over the npart partial sums of the route's row,
// in ascending order; with the gates g = softmax of the chosen logits,
// dlogits[t, ids[t, j]] = g_j (dgate_j - S), S = sum_j g_j dgate_j (fmaf in
// ascending slot order); every other logit's gradient is 0. One warp per
// token, lane j holding slot j.
namespace {
__global__ void __launch_bounds__(256) router_bwd_kernel(const float* __restrict__ part, int npart,
                                                         const int32_t* __restrict__ route_row,
                                                         const int32_t* __restrict__ ids,
                                                         const float* __restrict__ gates,
                                                         float* __restrict__ dlogits,
                                                         int64_t n_tokens, int E, int k,
                                                         int64_t rows_max, int32_t* dev_status) {
  const int lane = threadIdx.x & 31;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (t >= n_tokens) return;
  float dg = 0.0f, g = 0.0f;
  int id = -1, bad = 0;
  if (lane < k) {
    const int64_t rr = __ldg(route_row + t * k + lane);
    g = __ldg(gates + t * k + lane);
    id = __ldg(ids + t * k + lane);
    if (rr < 0 || rr >= rows_max || id < 0 || id >= E) {
      bad = 1;
    } else {
      const float* pr = part + rr * npart;
      for (int c = 0; c < npart; ++c) dg += __ldg(pr + c);
    }
  }
  float S = 0.0f;
  for (int j = 0; j < k; ++j)
    S = __fmaf_rn(__shfl_sync(0xFFFFFFFFu, g, j), __shfl_sync(0xFFFFFFFFu, dg, j), S);
  const float dl = g * (dg - S);
  float* out = dlogits + t * E;
  for (int e = lane; e < E; e += 32) out[e] = 0.0f;
  __syncwarp();  // orders the zeros before the k values written below
  if (lane < k && !bad) out[id] = dl;
  if (__any_sync(0xFFFFFFFFu, bad) && lane == 0) atomicOr(dev_status, MOE_DEV_BAD_SCHEDULE);
}
}  // namespace

cudaError_t launch_router_backward(const float* part, int32_t npart, const int32_t* route_row,
                                   const int32_t* ids, const float* gates, float* dlogits,
                                   int64_t n_tokens, int32_t E, int32_t k, int64_t rows_max,
                                   int32_t* dev_status, cudaStream_t s) {
  if (n_tokens == 0) return cudaSuccess;
  const int64_t blocks = (n_tokens + 7) / 8;
  router_bwd_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(part, npart, route_row, ids, gates,
                                                                 dlogits, n_tokens, E, k, rows_max,
                                                                 dev_status);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace moe
