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
// 32 at a time. Ranks inside a 32-route step come from a match mask (equal
// ids among the warp's lanes) and a popcount of the lower lanes; ranks across
// steps, warps and blocks from exclusive prefix sums of integer counts. The
// one-launch kernel adds the totals M with integer atomics, whose sum does not
// depend on their order: nothing is decided by the order of atomics, so Phi is
// deterministic and equal to the definition.
//
// One cooperative launch runs all four stages with one grid barrier when
// every block fits on the device at once (sched_fused_kernel, below);
// otherwise four kernels (one stream, no host round trip):
//   count    grid (C, P): per-block expert histogram -> ws[r][c][l]
//   scan     per (r, l): exclusive prefix over c in place; M[l][r] -> counts
//   offsets  one block: T[l] = sum_r M, Tp = ceil(T/pad)*pad, S = prefix(Tp)
//   scatter  grid (C, P): per-warp bases, then place every route once; pad
//            rows of Phi are filled with (-1,-1)
// Route reads: the four-kernel chain reads each route id in count and again
// in scatter (2*P*R, the pages' count); the one-launch kernel keeps a block's
// ids in registers between its phases and reads each once.
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

// The lanes of the warp whose key equals this lane's (keys in [0, 2^nbits)),
// built from one ballot per key bit: the same mask as __match_any_sync,
// at a fraction of its cost.
__device__ __forceinline__ unsigned match_by_ballots(int key, int nbits) {
  unsigned m = 0xFFFFFFFFu;
  for (int b = 0; b < nbits; ++b) {
    const bool bit = (key >> b) & 1;
    const unsigned v = __ballot_sync(0xFFFFFFFFu, bit);
    m &= bit ? v : ~v;
  }
  return m;
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

// ---------------------------------------------------------------- one launch
// The same four stages in one cooperative launch (every block resident at
// once), with one grid barrier:
//   A  each block (c, r) reads its 2,048 route ids once and keeps them in
//      registers; each warp builds the match masks of its 32-route steps from
//      ballots over the id bits, its expert histogram in shared memory and,
//      from the running histogram, each route's rank among the warp's routes
//      to its expert (kept in registers for C); the block writes its
//      histogram to ws[r][c][l] and adds the nonzero entries to the totals
//      M[l][r] with integer atomics;
//   |  the barrier
//   C  every block loads M and its own base, the sum of ws[r][c'][l] over
//      the peer's earlier blocks c' < c (rows 0..c-1 of the peer's slab),
//      computes T, Tp and S itself (block (0,0) writes offsets and counts),
//      derives its warps' bases from its block base, then places its routes
//      from the registers of phase A and fills its share of padding rows.
// Each route id is read from memory once. The barrier is a counter in ws,
// zero at launch with M (the routing kernel of a layer call zeroes them, a
// moe_schedule call with a memset): a block arrives with a release add and
// waits, with an acquire load, until all blocks of the launch arrived; the
// wait is bounded (timeout_ns), after which the block raises
// MOE_DEV_TIMEOUT and leaves without writing anything more.
struct FusedParams {
  SchedParams sp;
  uint32_t* bar;      // arrival counter, zero at launch
  int32_t* m;         // [E][P] route totals M, zero at launch (integer atomics)
  int32_t expect;     // blocks that must arrive (the grid; more only in the self test)
  int64_t timeout_ns;
};

// Row stride of the one-launch kernel's shared copy of M: P rounded up to
// whole 16-byte vectors, made an odd number of vectors.
__host__ __device__ __forceinline__ int m_row_stride(int P) {
  const int v = (P + 3) / 4;
  return 4 * (v % 2 ? v : v + 1);
}

__device__ __forceinline__ uint64_t sched_now_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Grid barrier number `gen` (1, 2, ...): true once every block of the launch
// arrived, false (MOE_DEV_TIMEOUT raised) if the wait gave up.
__device__ __forceinline__ bool sched_grid_barrier(const FusedParams& f, uint32_t gen) {
  __shared__ int s_ok;
  __syncthreads();
  if (threadIdx.x == 0) {
    int ok = 1;
    __threadfence();  // the block's writes (ordered before by the bar.sync above)
    asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(f.bar) : "memory");
    const uint32_t target = gen * static_cast<uint32_t>(f.expect);
    const uint64_t t0 = sched_now_ns();
    for (;;) {
      uint32_t v;
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(f.bar) : "memory");
      if (v >= target) break;
      if (sched_now_ns() - t0 > static_cast<uint64_t>(f.timeout_ns)) {
        atomicOr(f.sp.dev_status, MOE_DEV_TIMEOUT);
        ok = 0;
        break;
      }
      __nanosleep(64);
    }
    __threadfence();
    s_ok = ok;
  }
  __syncthreads();
  return s_ok != 0;
}

__global__ void __launch_bounds__(kThreads) sched_fused_kernel(FusedParams f) {
  const SchedParams& p = f.sp;
  extern __shared__ __align__(16) int32_t smem[];
  const int SP = m_row_stride(p.P);
  int32_t* s_m = smem;                   // [E][SP] M, zeros after column P
  int32_t* wbase = s_m + p.E * SP;       // [kWarps][E] warp counts, then warp bases
  int32_t* s_off = wbase + kWarps * p.E;  // [E+1] S
  int32_t* s_base = s_off + p.E + 1;     // [E] routes of earlier blocks of this peer
  __shared__ int32_t s_part[kThreads];
  const int c = blockIdx.x, r = blockIdx.y;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int R = p.Tm * p.k;
  const int E = p.E, P = p.P;

  // ---- A: count (ids read once, kept in registers)
  int32_t* wh = wbase + w * E;
  for (int l = lane; l < E; l += 32) wh[l] = 0;
  for (int l = threadIdx.x; l < E; l += kThreads) {
    s_base[l] = 0;
    for (int q = P; q < SP; ++q) s_m[l * SP + q] = 0;
  }
  __syncwarp();
  const int q0 = c * kSchedBlockRoutes + w * kWarpRoutes;
  // keys: the expert id, or E for a lane without a valid route. pre[s]: the
  // rank of step s's route among this warp's routes to its expert (routes of
  // earlier steps, then of lower lanes), taken from the running histogram
  // here so that the placement needs no running count of its own
  const int nbits = 32 - __clz(E);  // enough bits for 0..E
  const unsigned lower = (1u << lane) - 1u;
  int key[kSteps];
  int pre[kSteps];
  int bad = 0;
#pragma unroll
  for (int s = 0; s < kSteps; ++s) {
    const int q = q0 + s * 32 + lane;
    const int id = (q < R) ? __ldg(p.ids + route_index(p, r, q)) : -1;
    const bool ok = static_cast<unsigned>(id) < static_cast<unsigned>(E);
    if (q < R && !ok) bad = 1;
    key[s] = ok ? id : E;
  }
  if (bad) atomicOr(p.dev_status, MOE_DEV_BAD_EXPERT_ID);
#pragma unroll
  for (int s = 0; s < kSteps; ++s) {
    const unsigned m = match_by_ballots(key[s], nbits);
    const int lead = __ffs(m) - 1;  // first lane of this lane's key group
    int before = 0;
    if (key[s] != E && lane == lead) {
      before = wh[key[s]];
      wh[key[s]] = before + __popc(m);
    }
    pre[s] = __shfl_sync(kFull, before, lead) + __popc(m & lower);
    __syncwarp();
  }
  __syncthreads();
  {
    int32_t* out = p.ws + (static_cast<int64_t>(r) * p.C + c) * E;
    for (int l = threadIdx.x; l < E; l += kThreads) {
      int h = 0;
#pragma unroll
      for (int ww = 0; ww < kWarps; ++ww) h += wbase[ww * E + l];
      if (h) atomicAdd(f.m + l * P + r, h);  // M[l][r]: integer sums, any order
      out[l] = h;
    }
  }
  if (!sched_grid_barrier(f, 1)) return;

  // ---- C: M, this block's bases, offsets, warp bases, placement, padding
  // M (E * P words) and the block's bases are loaded in one round. The base
  // of expert l is the sum of H[r][c'][l] over the earlier blocks c' < c of
  // this peer: rows 0..c-1 of the peer's [C][E] slab, contiguous. Thread
  // (w, lane) takes experts lane + 32 j and rows w + 8 i (48 loads per round
  // for E <= 384 and c <= 32) and adds its sums into s_base with shared
  // atomics. M goes to shared memory as [E][SP] rows (m_row_stride): the
  // placement loop below reads a route's row as 16-byte vectors, and with an
  // odd number of vectors per row the rows of 8 unrelated ids start in
  // distinct groups of four banks.
  {
    const int n = E * P;
    int mv[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int i = threadIdx.x + u * kThreads;
      mv[u] = i < n ? __ldcg(f.m + i) : 0;
    }
    const int32_t* hb = p.ws + static_cast<int64_t>(r) * p.C * E;
    constexpr int kJ = 12, kI = 4;  // experts per lane, rows per warp in one round
    for (int j0 = 0; j0 < E; j0 += 32 * kJ) {
      for (int i0 = 0; i0 < c; i0 += kWarps * kI) {
        int hv[kJ][kI];
#pragma unroll
        for (int jj = 0; jj < kJ; ++jj)
#pragma unroll
          for (int ii = 0; ii < kI; ++ii) {
            const int l = j0 + lane + 32 * jj, cc = i0 + w + kWarps * ii;
            hv[jj][ii] = (l < E && cc < c) ? __ldcg(hb + static_cast<int64_t>(cc) * E + l) : 0;
          }
#pragma unroll
        for (int jj = 0; jj < kJ; ++jj) {
          const int l = j0 + lane + 32 * jj;
          int sum = 0;
#pragma unroll
          for (int ii = 0; ii < kI; ++ii) sum += hv[jj][ii];
          if (sum) atomicAdd(s_base + l, sum);
        }
      }
    }
    // (i / P, i % P) for i = threadIdx.x + u * kThreads, stepped without dividing
    int q = threadIdx.x / P, rem = threadIdx.x - (threadIdx.x / P) * P;
    const int sq = kThreads / P, sr = kThreads - (kThreads / P) * P;
    const bool first_block = blockIdx.x == 0 && blockIdx.y == 0;
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int i = threadIdx.x + u * kThreads;
      if (i < n) {
        s_m[q * SP + rem] = mv[u];
        if (first_block) p.counts[i] = mv[u];
      }
      q += sq;
      rem += sr;
      if (rem >= P) {
        rem -= P;
        ++q;
      }
    }
    for (int i = threadIdx.x + 16 * kThreads; i < n; i += kThreads) {  // E * P > 4,096
      const int v = __ldcg(f.m + i);
      s_m[(i / P) * SP + i % P] = v;
      if (first_block) p.counts[i] = v;
    }
  }
  __syncthreads();
  // padded totals Tp[l] into s_off, one expert per thread (its M row as vectors)
  for (int l = threadIdx.x; l < E; l += kThreads) {
    int T = 0;
    for (int q = 0; q < P; q += 4) {
      const int4 v = *reinterpret_cast<const int4*>(s_m + l * SP + q);
      T += v.x + v.y + v.z + v.w;
    }
    s_off[l] = (T + p.pad - 1) / p.pad * p.pad;
  }
  __syncthreads();
  {
    // thread t owns experts [4t, 4t + 4) (E <= 1024): a block-wide exclusive
    // scan of the per-thread sums of Tp, written over Tp
    const int l0 = threadIdx.x * 4;
    int tpv[4];
    int tsum = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int l = l0 + i;
      tpv[i] = l < E ? s_off[l] : 0;
      tsum += tpv[i];
    }
    int x = tsum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(kFull, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) s_part[w] = x;
    __syncthreads();
    int run = x - tsum;
    for (int ww = 0; ww < w; ++ww) run += s_part[ww];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int l = l0 + i;
      if (l < E) s_off[l] = run;
      run += tpv[i];
    }
    if (threadIdx.x == kThreads - 1) s_off[E] = run;  // the last thread's end: the total
  }
  __syncthreads();
  if (blockIdx.x == 0 && blockIdx.y == 0)
    for (int l = threadIdx.x; l <= E; l += kThreads) p.offsets[l] = s_off[l];

  // warp bases = block base (exclusive over blocks) + counts of earlier warps
  {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int l = threadIdx.x + u * kThreads;
      if (l >= E) break;
      int run = s_base[l];
#pragma unroll
      for (int ww = 0; ww < kWarps; ++ww) {
        const int v = wbase[ww * E + l];
        wbase[ww * E + l] = run;
        run += v;
      }
    }
  }
  __syncthreads();

  // the token of route q is q / k: one division, then stepped by 32 routes
  int tq = (q0 + lane) / p.k, tr = (q0 + lane) - tq * p.k;
  const int dq = 32 / p.k, dr = 32 - dq * p.k;
#pragma unroll
  for (int s = 0; s < kSteps; ++s) {
    const int q = q0 + s * 32 + lane;
    const int id = key[s];
    const bool valid = id != E;
    if (q < R) {
      const int64_t g = route_index(p, r, q);
      if (valid) {
        // o: the route's stable rank among peer r's routes to expert id
        const int o = wh[id] + pre[s];
        // columns past P hold zeros, which add nothing (o >= 0)
        int pos = 0;
        for (int q = 0; q < P; q += 4) {
          const int4 v = *reinterpret_cast<const int4*>(s_m + id * SP + q);
          pos += min(v.x, o) + min(v.y, o) + min(v.z, o) + min(v.w, o);
          pos += (q < r && v.x > o) + (q + 1 < r && v.y > o) + (q + 2 < r && v.z > o) +
                 (q + 3 < r && v.w > o);
        }
        const int row = s_off[id] + pos;
        reinterpret_cast<int2*>(p.phi)[row] = make_int2(r, p.t0 + tq);
        p.route_row[g] = row;
      } else {
        p.route_row[g] = -1;
      }
    }
    tq += dq;
    tr += dr;
    if (tr >= p.k) {
      tr -= p.k;
      ++tq;
    }
  }

  const int nb = gridDim.x * gridDim.y;
  const int b = blockIdx.y * gridDim.x + blockIdx.x;
  for (int l = b; l < E; l += nb) {
    int T = 0;
    for (int q = 0; q < P; q += 4) {
      const int4 v = *reinterpret_cast<const int4*>(s_m + l * SP + q);
      T += v.x + v.y + v.z + v.w;
    }
    const int start = s_off[l] + T, end = s_off[l + 1];
    for (int row = start + threadIdx.x; row < end; row += kThreads)
      reinterpret_cast<int2*>(p.phi)[row] = make_int2(-1, -1);
  }
}

inline int32_t blocks_per_peer(int32_t Tm, int32_t k) {
  const int64_t R = static_cast<int64_t>(Tm) * k;
  return static_cast<int32_t>((R + kSchedBlockRoutes - 1) / kSchedBlockRoutes);
}

}  // namespace

// [P][C][E] block counters; then, on a 64-byte boundary, the one-launch
// path's barrier counter (alone on its line) and its [E][P] totals M.
static int64_t counter_words(int32_t P, int32_t N, int32_t k, int32_t E) {
  const int64_t C = blocks_per_peer(N, k);
  return static_cast<int64_t>(P) * (C > 0 ? C : 1) * E;
}

static int64_t barrier_offset(int32_t P, int32_t N, int32_t k, int32_t E) {
  return (counter_words(P, N, k, E) + 15) / 16 * 16;
}

size_t schedule_ws_bytes(int32_t P, int32_t N, int32_t k, int32_t E) {
  const int64_t words = barrier_offset(P, N, k, E) + 16 + static_cast<int64_t>(E) * P;
  return static_cast<size_t>(words) * sizeof(int32_t);
}

namespace {

// Shared memory of the one-launch kernel: M [E][m_row_stride(P)], warp
// counts [8][E], S [E+1], block bases [E].
size_t fused_smem_bytes(int32_t P, int32_t E) {
  return (static_cast<size_t>(E) * m_row_stride(P) + static_cast<size_t>(kWarps) * E + E + 1 +
          E) *
         sizeof(int32_t);
}

// Whether the one-launch kernel can run for this grid: its shared memory fits
// and every block can be resident at once (a cooperative launch requires it).
bool fused_fits(int32_t C, int32_t P, int32_t E) {
  const size_t smem = fused_smem_bytes(P, E);
  if (C <= 0 || smem > 100 * 1024) return false;
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(sched_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return false;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, sched_fused_kernel, kThreads, smem) !=
      cudaSuccess)
    return false;
  return static_cast<int64_t>(per_sm) * device_sm_count() >= static_cast<int64_t>(C) * P;
}

cudaError_t launch_fused(const SchedParams& p, int32_t extra_expect, int64_t timeout_ns,
                         cudaStream_t s, bool barrier_zeroed) {
  FusedParams f;
  f.sp = p;
  int32_t* bar = p.ws + barrier_offset(p.P, p.N, p.k, p.E);
  f.bar = reinterpret_cast<uint32_t*>(bar);
  f.m = bar + 16;
  f.expect = p.C * p.P + extra_expect;
  f.timeout_ns = timeout_ns;
  cudaError_t e = cudaSuccess;
  if (!barrier_zeroed &&
      (e = cudaMemsetAsync(bar, 0, sizeof(int32_t) * (16 + static_cast<size_t>(p.E) * p.P), s)) !=
          cudaSuccess)
    return e;
  cudaLaunchAttribute coop[1];
  coop[0].id = cudaLaunchAttributeCooperative;
  coop[0].val.cooperative = 1;
  cudaLaunchConfig_t c = {};
  c.gridDim = dim3(p.C, p.P);
  c.blockDim = dim3(kThreads);
  c.dynamicSmemBytes = fused_smem_bytes(p.P, p.E);
  c.stream = s;
  c.attrs = coop;
  c.numAttrs = 1;
  e = cudaLaunchKernelEx(&c, sched_fused_kernel, f);
  note_launches(1);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

SchedParams make_params(const int32_t* ids, const moe_shape_t& sh, Slice sl, int32_t* phi,
                        int32_t* offsets, int32_t* counts, int32_t* route_row, int32_t* ws,
                        int32_t* dev_status) {
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
  return p;
}

}  // namespace

cudaError_t launch_schedule_barrier_selftest(const int32_t* ids, const moe_shape_t& sh,
                                             int32_t* phi, int32_t* offsets, int32_t* counts,
                                             int32_t* route_row, int32_t* ws, int32_t* dev_status,
                                             int64_t timeout_ns, cudaStream_t s) {
  const SchedParams p =
      make_params(ids, sh, Slice{0, sh.N}, phi, offsets, counts, route_row, ws, dev_status);
  if (!fused_fits(p.C, p.P, p.E)) return cudaErrorInvalidConfiguration;
  return launch_fused(p, /*extra_expect=*/1, timeout_ns, s, false);
}

int32_t* schedule_barrier_word(int32_t* ws, const moe_shape_t& sh) {
  return ws + barrier_offset(sh.P, sh.N, sh.k, sh.E);
}

int32_t schedule_zero_words(const moe_shape_t& sh) { return 16 + sh.E * sh.P; }

cudaError_t launch_schedule(const int32_t* ids, const moe_shape_t& sh, Slice sl, int32_t* phi,
                            int32_t* offsets, int32_t* counts, int32_t* route_row, int32_t* ws,
                            int32_t* dev_status, cudaStream_t s, bool barrier_zeroed) {
  const SchedParams p = make_params(ids, sh, sl, phi, offsets, counts, route_row, ws, dev_status);
  // one launch when every block fits on the device at once (the Kimi shape:
  // 28 x 8 blocks); otherwise the four-kernel chain below
  if (fused_fits(p.C, p.P, p.E)) return launch_fused(p, 0, kWaitTimeoutNs, s, barrier_zeroed);
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
