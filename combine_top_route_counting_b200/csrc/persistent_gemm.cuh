// Pieces shared by the persistent, warp-specialised grouped GEMMs (the
// forward FFN in expert_ffn.cu and its backward in expert_ffn_bwd.cu):
// thread roles, the per-expert segment table, the tile-id ring that hands
// tiles out dynamically, and the grouped row raster.
//
// One CTA (or CTA pair) per SM, 384 threads:
//   warp 0      TMA producer
//   warp 1      TMEM allocator and MMA issuer
//   warp 2      tile scheduler (lane 0 of the pair's leader)
//   warp 3      spare (the gather-fed GEMM1 uses it as a second producer)
//   warps 4-11  epilogue
#pragma once

#include <cuda_bf16.h>

#include "internal.cuh"
#include "sm100.cuh"

namespace moe {
namespace pg {

constexpr int kNumThreads = 384;
constexpr int kEpiWarp0 = 4;
constexpr int kNumEpiWarps = 8;
constexpr int kTmemCols = 512;  // 2 accumulators x 256 fp32 columns
constexpr int kUmmaK = 16;      // K of one bf16 tcgen05.mma
constexpr int kRing = 4;        // tile ids in flight between the scheduler and the roles

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat16 a = __float2bfloat16_rn(lo);
  const __nv_bfloat16 b = __float2bfloat16_rn(hi);
  return static_cast<uint32_t>(__bfloat16_as_ushort(a)) |
         (static_cast<uint32_t>(__bfloat16_as_ushort(b)) << 16);
}

// Per-expert segment table in shared memory: s_off[0..E] = the segment
// starts; s_end[l] = the end of expert l's real rows (its routes counted from
// counts, else the whole segment). Sets *bad_flag when a segment bound is not
// a multiple of bm, decreases, passes rows_max, or counts exceed a segment.
// Called by every thread of the CTA (it synchronises once).
__device__ __forceinline__ void load_segments(const int32_t* offsets, const int32_t* counts, int E,
                                              int P, int bm, int64_t rows_max, int32_t* s_off,
                                              int32_t* s_end, int* bad_flag) {
  const int tid = threadIdx.x, nthreads = blockDim.x;
  for (int l = tid; l <= E; l += nthreads) s_off[l] = __ldg(offsets + l);
  __syncthreads();
  for (int l = tid; l < E; l += nthreads) {
    const int a = s_off[l], b = s_off[l + 1];
    bool bad = a < 0 || b < a || (a % bm) || (b % bm) || b > rows_max;
    int T = b - a;
    if (counts) {
      int t = 0;
      for (int r = 0; r < P; ++r) t += __ldg(counts + l * P + r);
      if (t < 0 || t > b - a) bad = true;
      else T = t;
    }
    if (bad) *bad_flag = 1;
    s_end[l] = a + T;
  }
}

// The tile-id ring: the leader's scheduler thread takes tile ids from a
// device-wide counter and posts them, in order, to a kRing-deep ring in the
// shared memory of both CTAs of a pair; every consuming role reads the same
// sequence. CTAs that run ahead simply take more tiles, so the tiles in
// flight stay a narrow window of consecutive ids and the operands they share
// are still in L2.
struct TileRing {
  int* ring;               // [kRing] tile ids (this CTA's copy)
  uint32_t full0;          // TID_FULL[0] barrier of this CTA
  uint32_t empty_local;    // TID_EMPTY[0] of this CTA
  uint32_t empty_leader;   // TID_EMPTY[0] of the pair's leader (shared::cluster)
  bool follower;           // a follower releases its slots on the leader

  // The next id of this role's sequence: -1 at the end, -2 if a wait gave
  // up. One thread per consuming warp calls it. The slot is released with a
  // release-ordered arrive (the read of the id must not move after it): CTA
  // scope for the leader's own roles, cluster scope for the follower's,
  // whose arrive is remote.
  template <bool PAIR>
  __device__ __forceinline__ int next(int& pos, uint32_t& ph, const sm100::WaitCtx& wc) const {
    const int j = pos % kRing;
    if (!sm100::wait_bounded<PAIR>(full0 + j * 8, ph, wc)) return -2;
    const int t = reinterpret_cast<volatile int*>(ring)[j];
    if (PAIR && follower) sm100::mbar_arrive_cluster(empty_leader + j * 8);
    else sm100::mbar_arrive(empty_local + j * 8);
    if (++pos % kRing == 0) ph ^= 1u;
    return t;
  }

  // The scheduler (lane 0 of warp 2 of the leader): hands out ids 0..num_tiles-1
  // from *counter, then -1. With a pair it also writes the follower's ring.
  template <bool PAIR>
  __device__ __forceinline__ void schedule(int* counter, int num_tiles,
                                           const sm100::WaitCtx& wc) const {
    const uint32_t ring_peer = PAIR ? sm100::mapa_shared(sm100::smem_u32(ring), 1) : 0u;
    const uint32_t full_peer = PAIR ? sm100::mapa_shared(full0, 1) : 0u;
    uint32_t eph = 0;
    for (int i = 0;; ++i) {
      const int j = i % kRing;
      if (!sm100::wait_bounded<PAIR>(empty_local + j * 8, eph ^ 1u, wc)) break;
      int t = atomicAdd(counter, 1);
      if (t >= num_tiles) t = -1;
      reinterpret_cast<volatile int*>(ring)[j] = t;
      sm100::mbar_arrive(full0 + j * 8);
      if (PAIR) {
        sm100::st_shared_cluster_u32(ring_peer + j * 4, static_cast<uint32_t>(t));
        sm100::mbar_arrive_cluster(full_peer + j * 8);
      }
      if (j == kRing - 1) eph ^= 1u;
      if (t < 0) break;
    }
  }
};

// Row-grouped tiles (M = the experts' rows, tiles_n column blocks): tile ->
// (first row, column block, expert); false if the tile holds only padding.
// Tiles are numbered expert by expert (expert l owns tiles
// [S[l]/BM * tiles_n, S[l+1]/BM * tiles_n)) and, inside an expert, in a
// grouped raster: chunks of up to RM M-tiles; inside a chunk, groups of RN
// column blocks; inside a group, columns fastest. The expert comes from a
// binary search over the segment starts.
template <int BM, int RM, int RN>
__device__ __forceinline__ bool grouped_row_tile(int tile, const int32_t* s_off,
                                                 const int32_t* s_end, int E, int tiles_n,
                                                 int& row0, int& n, int& l) {
  const int u = tile / tiles_n;  // the tile's position in M-tile units
  int lo = 0, hi = E - 1;        // expert: largest l with S[l]/BM <= u
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s_off[mid] / BM <= u) lo = mid;
    else hi = mid - 1;
  }
  l = lo;
  const int m0 = s_off[l] / BM;
  const int mcount = s_off[l + 1] / BM - m0;  // >= 1 for the expert owning u
  const int j = tile - m0 * tiles_n;           // index inside the expert
  const int mc = j / (RM * tiles_n);           // M chunk
  const int rows = min(RM, mcount - mc * RM);  // M-tiles in this chunk
  const int jj = j - mc * RM * tiles_n;
  const int ng = jj / (rows * RN);             // column group
  const int gsize = min(RN, tiles_n - ng * RN);
  const int rr = jj - ng * rows * RN;
  const int m = rr / gsize;
  n = ng * RN + (rr - m * gsize);
  row0 = (m0 + mc * RM + m) * BM;
  return row0 < s_end[l];
}

// Wait (bounded, acquire at GPU scope) until *flag != 0: a landed-dispatch
// producer's wait for a block of gathered rows that another CTA's warp lands.
// Gives up like wait_bounded: after timeout_ns, or once another role of the
// CTA gave up.
__device__ __forceinline__ bool wait_flag_bounded(const int* flag, const sm100::WaitCtx& w) {
  auto ready = [&]() {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(flag) : "memory");
    return v != 0;
  };
  if (ready()) return true;
  const uint64_t t0 = sm100::globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    __nanosleep(32);
    if (ready()) return true;
    if ((it & 15u) == 0) {
      if (*w.abort) return false;
      if (sm100::globaltimer_ns() - t0 > static_cast<uint64_t>(w.timeout_ns)) {
        *w.abort = 1;
        atomicOr(w.dev_status, w.timeout_flag);
        return false;
      }
    }
  }
}

// A launch's tile counter is two words: the next tile id, and the CTAs that
// have finished. Called once per CTA (one thread, after the CTA's last use of
// the counter): the last CTA to finish puts both words back to zero, so the
// counter is clean for whichever launch takes it next, whenever that runs.
__device__ __forceinline__ void finish_tile_counter(int* counter) {
  __threadfence();  // this CTA's tile fetches come before its count
  if (atomicAdd(counter + 1, 1) == static_cast<int>(gridDim.x) - 1) {
    __threadfence();  // every CTA's fetches come before the reset
    atomicExch(counter, 0);
    atomicExch(counter + 1, 0);
  }
}

// Launch a persistent kernel on every SM: `cg` CTAs per cluster (1 or 2),
// 384 threads, `smem` bytes of dynamic shared memory.
template <class... KArgs, class... Args>
cudaError_t launch_persistent(void (*kernel)(KArgs...), int cg, size_t smem, cudaStream_t s,
                              Args&&... args) {
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int sms = device_sm_count();
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.gridDim = dim3(cg == 2 ? (sms / 2) * 2 : sms);
  cfg.blockDim = dim3(kNumThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  if (cg == 2) {
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  note_launches(1);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace pg
}  // namespace moe
