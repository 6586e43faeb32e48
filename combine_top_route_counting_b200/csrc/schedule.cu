// Step 2: the pull-dispatch schedule table Phi as a single-pass counting sort.
//
// "Scan once, scatter once", section "The fix is a counting sort": count
// routes per expert, peer and scheduler thread; prefix the per-thread counts;
// pad each expert segment and compute its base row; scatter each route once.
// "Mixture-of-Kittens: A MoE Megakernel for GB300 NVL72", section 2
// (on-device schedule generation): route (r, o) of expert l lands at
// Phi[S[l] + p], p = sum_{r'} min(M[l,r'], o) + |{r' < r : M[l,r'] > o}|,
// o being the route's stable rank among peer r's routes to expert l.
//
// The stable order within (expert, peer) is ascending route index q. The
// pages spread a peer's routes over 1,024 logical threads with contiguous
// chunks; any contiguous decomposition gives the same order, so here a block
// owns 2,048 consecutive routes and each of its 8 warps 256 of them, consumed
// 32 at a time. Ranks inside a 32-route step come from __match_any_sync and a
// popcount of the lower lanes; ranks across steps, warps and blocks from
// exclusive prefix sums of integer counts. Nothing is decided by the order of
// atomics, so Phi is deterministic and equal to the definition.
//
// Kernels (one stream, no host round trip):
//   count    grid (C, P): per-block expert histogram -> ws[r][c][l]
//   scan     per (r, l): exclusive prefix over c in place; M[l][r] -> counts
//   offsets  one block: T[l] = sum_r M, Tp = ceil(T/pad)*pad, S = prefix(Tp)
//   scatter  grid (C, P): per-warp bases, then place every route once; pad
//            rows of Phi are filled with (-1,-1)
// Route reads: each route id is read by count and by scatter (2*P*R).
#include "internal.cuh"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = 8;
constexpr int kWarpRoutes = 256;
constexpr int kSteps = kWarpRoutes / 32;
constexpr int kInvalid = 0x40000000;  // match key of lanes without a valid route
constexpr unsigned kFull = 0xFFFFFFFFu;
static_assert(kWarps * kWarpRoutes == kSchedBlockRoutes, "block covers 2048 routes");

// Programmatic dependent launch: a kernel of the chain lets the next one be
// scheduled early (launch_dependents) and waits for its predecessor's results
// before touching them (wait). Every block executes the wait unconditionally,
// so each kernel completes after its predecessor.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

struct SchedParams {
  const int32_t* ids;
  int32_t P, N, k, E, pad;
  int32_t t0, Tm;  // token slice of every peer
  int32_t C;       // counting blocks per peer
  int32_t* phi;
  int32_t* offsets;
  int32_t* counts;
  int32_t* route_row;
  int32_t* ws;     // [P][C][E] counts, then exclusive block bases
  int32_t* dev_status;
};

__device__ __forceinline__ int64_t route_index(const SchedParams& p, int r, int q) {
  return (static_cast<int64_t>(r) * p.N + p.t0) * p.k + q;
}

__global__ void __launch_bounds__(kThreads) sched_count_kernel(SchedParams p) {
  extern __shared__ int32_t hist[];
  pdl_launch_dependents();
  const int c = blockIdx.x, r = blockIdx.y;
  const int R = p.Tm * p.k;
  for (int l = threadIdx.x; l < p.E; l += kThreads) hist[l] = 0;
  __syncthreads();
  int bad = 0;
#pragma unroll
  for (int s = 0; s < kSchedBlockRoutes / kThreads; ++s) {
    const int q = c * kSchedBlockRoutes + s * kThreads + threadIdx.x;
    if (q < R) {
      const int id = __ldg(p.ids + route_index(p, r, q));
      if (static_cast<unsigned>(id) < static_cast<unsigned>(p.E))
        atomicAdd(&hist[id], 1);  // integer counts: order-independent
      else
        bad = 1;
    }
  }
  if (bad) atomicOr(p.dev_status, MOE_DEV_BAD_EXPERT_ID);
  __syncthreads();
  int32_t* out = p.ws + (static_cast<int64_t>(r) * p.C + c) * p.E;
  for (int l = threadIdx.x; l < p.E; l += kThreads) out[l] = hist[l];
}

__global__ void __launch_bounds__(kThreads) sched_scan_kernel(SchedParams p) {
  pdl_launch_dependents();
  pdl_wait();
  const int idx = blockIdx.x * kThreads + threadIdx.x;
  if (idx >= p.P * p.E) return;
  const int r = idx / p.E, l = idx - r * p.E;
  int32_t* col = p.ws + static_cast<int64_t>(r) * p.C * p.E + l;
  const int64_t stride = p.E;
  int run = 0;
  int c = 0;
  for (; c + 8 <= p.C; c += 8) {  // eight independent loads in flight
    int v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = col[(c + u) * stride];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      col[(c + u) * stride] = run;
      run += v[u];
    }
  }
  for (; c < p.C; ++c) {
    const int v = col[c * stride];
    col[c * stride] = run;
    run += v;
  }
  p.counts[l * p.P + r] = run;
}

// One block of 1024 threads (E <= 1024): one expert per thread.
__global__ void __launch_bounds__(1024) sched_offsets_kernel(SchedParams p) {
  __shared__ int32_t warp_tot[32];
  pdl_launch_dependents();
  pdl_wait();
  const int l = threadIdx.x, lane = l & 31, w = l >> 5;
  int tp = 0;
  if (l < p.E) {
    int T = 0;
    for (int r = 0; r < p.P; ++r) T += p.counts[l * p.P + r];
    tp = (T + p.pad - 1) / p.pad * p.pad;
  }
  int x = tp;  // inclusive warp scan
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(kFull, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[w] = x;
  __syncthreads();
  if (w == 0) {
    int t = warp_tot[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(kFull, t, o);
      if (lane >= o) t += y;
    }
    warp_tot[lane] = t;  // inclusive over warps
  }
  __syncthreads();
  const int incl = x + (w > 0 ? warp_tot[w - 1] : 0);
  if (l < p.E) p.offsets[l] = incl - tp;
  if (l == 1023) p.offsets[p.E] = incl;  // tp = 0 beyond E: total
}

// STAGE: counts [E][P] and offsets [E+1] are copied to shared memory (when
// they fit), so the O(P) placement loop reads them from there.
template <bool STAGE>
__global__ void __launch_bounds__(kThreads) sched_scatter_kernel(SchedParams p) {
  extern __shared__ int32_t smem[];
  int32_t* wbase = smem;                      // [kWarps][E]
  int32_t* s_cnt = smem + kWarps * p.E;       // [E][P]   (STAGE)
  int32_t* s_off = s_cnt + p.E * p.P;         // [E+1]    (STAGE)
  const int c = blockIdx.x, r = blockIdx.y;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int R = p.Tm * p.k;
  int32_t* wh = wbase + w * p.E;
  for (int l = lane; l < p.E; l += 32) wh[l] = 0;
  __syncwarp();

  // pass 1: this warp's per-expert counts over its 256 routes (ids were
  // written before this chain started)
  const int q0 = c * kSchedBlockRoutes + w * kWarpRoutes;
  int key[kSteps];
#pragma unroll
  for (int s = 0; s < kSteps; ++s) {
    const int q = q0 + s * 32 + lane;
    const int id = (q < R) ? __ldg(p.ids + route_index(p, r, q)) : -1;
    key[s] = (static_cast<unsigned>(id) < static_cast<unsigned>(p.E)) ? id : kInvalid;
  }
#pragma unroll
  for (int s = 0; s < kSteps; ++s) {
    const unsigned m = __match_any_sync(kFull, key[s]);
    if (key[s] != kInvalid && lane == __ffs(m) - 1) wh[key[s]] += __popc(m);
    __syncwarp();
  }
  pdl_wait();  // block bases, counts and offsets come from the previous kernels
  const int32_t* cnt = p.counts;
  const int32_t* off = p.offsets;
  if (STAGE) {
    for (int i = threadIdx.x; i < p.E * p.P; i += kThreads) s_cnt[i] = p.counts[i];
    for (int i = threadIdx.x; i <= p.E; i += kThreads) s_off[i] = p.offsets[i];
    cnt = s_cnt;
    off = s_off;
  }
  __syncthreads();

  // per-warp bases = block base (prefix over blocks) + counts of earlier warps
  const int32_t* blk = p.ws + (static_cast<int64_t>(r) * p.C + c) * p.E;
  for (int l = threadIdx.x; l < p.E; l += kThreads) {
    int run = blk[l];
#pragma unroll
    for (int ww = 0; ww < kWarps; ++ww) {
      const int v = wbase[ww * p.E + l];
      wbase[ww * p.E + l] = run;
      run += v;
    }
  }
  __syncthreads();

  // pass 2: place every route once
  const unsigned lower = (1u << lane) - 1u;
#pragma unroll
  for (int s = 0; s < kSteps; ++s) {
    const int q = q0 + s * 32 + lane;
    const int id = key[s];
    const bool valid = id != kInvalid;
    const unsigned m = __match_any_sync(kFull, id);
    int o = 0;
    if (valid) o = wh[id] + __popc(m & lower);
    __syncwarp();
    if (valid && lane == __ffs(m) - 1) wh[id] += __popc(m);
    __syncwarp();
    if (q < R) {
      const int64_t g = route_index(p, r, q);
      if (valid) {
        const int32_t* Ml = cnt + id * p.P;
        int pos = 0;
        for (int r2 = 0; r2 < p.P; ++r2) {
          const int mm = Ml[r2];
          pos += min(mm, o);
          pos += (r2 < r && mm > o) ? 1 : 0;
        }
        const int row = off[id] + pos;
        reinterpret_cast<int2*>(p.phi)[row] = make_int2(r, p.t0 + q / p.k);
        p.route_row[g] = row;
      } else {
        p.route_row[g] = -1;  // invalid id: reported by the count kernel
      }
    }
  }

  // padding rows of the experts this block is responsible for
  const int nb = gridDim.x * gridDim.y;
  const int b = blockIdx.y * gridDim.x + blockIdx.x;
  for (int l = b; l < p.E; l += nb) {
    int T = 0;
    for (int r2 = 0; r2 < p.P; ++r2) T += cnt[l * p.P + r2];
    const int start = off[l] + T, end = off[l + 1];
    for (int row = start + threadIdx.x; row < end; row += kThreads)
      reinterpret_cast<int2*>(p.phi)[row] = make_int2(-1, -1);
  }
}

inline int32_t blocks_per_peer(int32_t Tm, int32_t k) {
  const int64_t R = static_cast<int64_t>(Tm) * k;
  return static_cast<int32_t>((R + kSchedBlockRoutes - 1) / kSchedBlockRoutes);
}

}  // namespace

size_t schedule_ws_bytes(int32_t P, int32_t N, int32_t k, int32_t E) {
  const int64_t C = blocks_per_peer(N, k);
  const int64_t words = static_cast<int64_t>(P) * (C > 0 ? C : 1) * E;
  return static_cast<size_t>(words) * sizeof(int32_t);
}

cudaError_t launch_schedule(const int32_t* ids, const moe_shape_t& sh, Slice sl, int32_t* phi,
                            int32_t* offsets, int32_t* counts, int32_t* route_row, int32_t* ws,
                            int32_t* dev_status, cudaStream_t s) {
  SchedParams p;
  p.ids = ids;
  p.P = sh.P;
  p.N = sh.N;
  p.k = sh.k;
  p.E = sh.E;
  p.pad = sh.pad;
  p.t0 = sl.t0;
  p.Tm = sl.Tm;
  p.C = blocks_per_peer(sl.Tm, sh.k);
  p.phi = phi;
  p.offsets = offsets;
  p.counts = counts;
  p.route_row = route_row;
  p.ws = ws;
  p.dev_status = dev_status;
  int launched = 0;
  cudaError_t e = cudaSuccess;
  // count runs in plain stream order (after whatever wrote ids); scan, offsets
  // and scatter are launched as programmatic dependents of their predecessor.
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  auto cfg = [&](dim3 grid, dim3 block, size_t smem, bool dependent) {
    cudaLaunchConfig_t c = {};
    c.gridDim = grid;
    c.blockDim = block;
    c.dynamicSmemBytes = smem;
    c.stream = s;
    c.attrs = dependent ? pdl : nullptr;
    c.numAttrs = dependent ? 1 : 0;
    return c;
  };
  if (p.C > 0) {
    const cudaLaunchConfig_t c = cfg(dim3(p.C, p.P), dim3(kThreads), p.E * sizeof(int32_t), false);
    e = cudaLaunchKernelEx(&c, sched_count_kernel, p);
    ++launched;
  }
  if (e == cudaSuccess) {
    const int scan_blocks = (p.P * p.E + kThreads - 1) / kThreads;
    const cudaLaunchConfig_t c = cfg(dim3(scan_blocks), dim3(kThreads), 0, p.C > 0);
    e = cudaLaunchKernelEx(&c, sched_scan_kernel, p);
    ++launched;
  }
  if (e == cudaSuccess) {
    const cudaLaunchConfig_t c = cfg(dim3(1), dim3(1024), 0, true);
    e = cudaLaunchKernelEx(&c, sched_offsets_kernel, p);
    ++launched;
  }
  if (e == cudaSuccess && p.C > 0) {
    const size_t stage_words = static_cast<size_t>(p.E) * p.P + p.E + 1;
    const bool stage = stage_words <= 8192;
    const size_t smem = (kWarps * static_cast<size_t>(p.E) + (stage ? stage_words : 0)) * 4;
    const cudaLaunchConfig_t c = cfg(dim3(p.C, p.P), dim3(kThreads), smem, true);
    e = stage ? cudaLaunchKernelEx(&c, sched_scatter_kernel<true>, p)
              : cudaLaunchKernelEx(&c, sched_scatter_kernel<false>, p);
    ++launched;
  }
  note_launches(launched);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace moe
