// Step 3b: grouped SwiGLU expert FFN on the 5th-generation tensor cores.
//
// "Mixture-of-Kittens: A MoE Megakernel for GB300 NVL72", section 5 (routed
// expert grouped GEMMs with SwiGLU fused) and section 3 (128x256 output
// tiles; the up/gate projections run side by side, the down projection is
// bounded by H). For each expert l, rows [S[l], S[l+1]) of the gathered
// buffer are multiplied by that expert's weights:
//   GEMM1: acc = xg . [W1[l] | W3[l]]  (fp32 in TMEM),
//          h = bf16_rne(silu(acc_W1) * acc_W3)
//   GEMM2: y = h . W2[l]  (fp32)
//
// Design (persistent, one CTA per SM, 384 threads, warp-specialised):
//   warp 0      TMA producer: ring of {A 128x64, B 64 x (256/CG)} bf16 tiles,
//               128-byte swizzle, mbarrier complete_tx
//   warp 1      TMEM allocator and MMA issuer: tcgen05.mma kind::f16, K=16,
//               A K-major, B MN-major (the weights are stored [K, N] with N
//               contiguous, so no transpose is needed)
//   warps 4-11  epilogue: tcgen05.ld of the fp32 accumulator (one TMEM lane per
//               row, two warps per lane quarter splitting the columns),
//               SwiGLU or fp32, 32-byte vector stores
//   TMEM        2 x 256 fp32 columns: the accumulator of tile i+1 fills while
//               the epilogue drains tile i
// Two geometries (CG = CTAs per MMA):
//   CG = 2 (segments padded to multiples of 256, the pages' padding): a
//     cluster of two CTAs on two SMs computes a 256x256 tile with
//     tcgen05.mma.cta_group::2 (M=256, N=256): each CTA loads its 128 rows of
//     A and 128 of the 256 B columns, so each SM moves half the operand bytes
//     per flop of a single-SM 128x256 tile. 6-stage ring of 32 KB.
//   CG = 1 (segments multiples of 128 only): 128x256 tile per CTA with
//     cta_group::1, 4-stage ring of 48 KB.
// GEMM1's B tile is [W1 cols | W3 cols] of the same 128 h columns, so one
// N=256 MMA produces both halves of SwiGLU (with CG = 2, CTA 0 holds the W1
// half and CTA 1 the W3 half). A tile never straddles two experts because
// every segment is a multiple of the tile height; the expert of a tile comes
// from a binary search over the segment offsets held in shared memory. Tiles
// holding only padding rows are skipped. Tiles are handed out dynamically in
// an expert-by-expert, N-block-major order, so the CTAs running at one time
// share an expert's A rows and a few weight column blocks through L2.
//
// Every output element is produced by one CTA with a fixed K order (no
// split-K, no atomics): the result is bitwise deterministic and independent
// of which other rows share the launch.
//
// Every mbarrier wait is bounded (sm100.cuh): if any wait gives up, all roles
// unwind, in-flight TMA loads and MMAs are drained with a bounded wait, TMEM
// is freed and MOE_DEV_TIMEOUT is raised.
#include <cuda_bf16.h>

#include "internal.cuh"
#include "persistent_gemm.cuh"
#include "sm100.cuh"

namespace moe {
namespace {

using namespace sm100;
using namespace pg;

// Tile geometry for CG CTAs per MMA (1: one SM, 2: a CTA pair on two SMs).
// TMA_STORE (GEMM2 on CTA pairs): the fp32 epilogue stages each warp's 32x16
// blocks in 64-byte-swizzled shared memory (2 KB per warp) and writes each
// with one TMA store, keeping the load/store unit free; the 16 KB of staging
// leave room for six pipeline stages, as GEMM1 has.
template <int CG, int MODE>
struct Cfg {
  static constexpr bool TMA_STORE = (CG == 2 && MODE == 1);
  static constexpr int STAGING_BYTES = TMA_STORE ? 8 * 2048 : 0;  // 8 warps x 32x16 fp32
  static constexpr int BM = 128 * CG;      // rows per tile (each CTA holds 128)
  static constexpr int BN = 256;           // accumulator columns per tile
  static constexpr int BK = 64;            // K per stage: one 128-byte swizzle row of bf16
  static constexpr int B_ATOMS = BN / CG / 64;   // 64-column B boxes held per CTA
  static constexpr int A_BYTES = 128 * BK * 2;   // 16 KB
  static constexpr int B_ATOM_BYTES = 64 * BK * 2;  // 8 KB
  static constexpr int STAGE_BYTES = A_BYTES + B_ATOMS * B_ATOM_BYTES;  // 48 / 32 KB
  static constexpr int STAGES = CG == 1 ? 4 : 6;
  static constexpr uint32_t IDESC = idesc_bf16_f32(BM, BN, /*B MN-major*/ 1);
  static constexpr int BAR_FULL = 0;
  static constexpr int BAR_EMPTY = STAGES;
  static constexpr int BAR_TFULL = 2 * STAGES;
  static constexpr int BAR_TEMPTY = 2 * STAGES + 2;
  static constexpr int BAR_DRAIN = 2 * STAGES + 4;
  static constexpr int BAR_TID_FULL = 2 * STAGES + 5;   // [kRing] tile id posted
  static constexpr int BAR_TID_EMPTY = 2 * STAGES + 9;  // [kRing] tile id consumed
  static constexpr int NUM_BARS = 2 * STAGES + 13;
  // consumers of each tile id: producer, MMA issuer and 8 epilogue warps of
  // the leader; producer and 8 epilogue warps of the follower
  static constexpr int TID_CONSUMERS = CG == 2 ? 19 : 10;
  static_assert(STAGE_BYTES % 1024 == 0 && A_BYTES % 1024 == 0, "swizzle atoms stay 1024-aligned");
};

struct FfnParams {
  int* tile_counter;       // {next tile to hand out, CTAs finished}; zero at launch
  const int2* phi;         // [rows_max] (src_rank, src_idx): GATHER only
  int32_t n_per_peer;      // N (GATHER: token row = src_rank * N + src_idx)
  const int32_t* offsets;  // [E+1]
  const int32_t* counts;   // [E, P] or null
  int32_t E, P;
  int32_t K;               // reduction length (H for GEMM1, I for GEMM2)
  int32_t Nout;            // output row length (I for GEMM1, H for GEMM2)
  int64_t rows_max;
  void* out;               // bf16 h [rows_max, I] or fp32 y [rows_max, H]
  int32_t* dev_status;
  int64_t timeout_ns;
  uint16_t* ab;            // SAVE_AB: bf16 pre-activations [rows_max, 2I], a | b
  const void* x;           // GATHER, LAND: token activations bf16 [P*N, H]
  uint16_t* xg;            // LAND: the gathered buffer [rows_max, H] the A map reads
  int* land_next;          // LAND: next 128-row block to land (0 at launch)
  int* land_ready;         // LAND: [rows_max / 128] block-landed flags (0 at launch)
};

template <int CG, int MODE>
size_t smem_bytes_for(int E) {
  using C = Cfg<CG, MODE>;
  return 1024 /*alignment slack*/ + static_cast<size_t>(C::STAGES) * C::STAGE_BYTES +
         C::STAGING_BYTES + C::NUM_BARS * 8 + 16 + kRing * 4 + static_cast<size_t>(2 * E + 1) * 4;
}

__device__ __forceinline__ float silu(float a) { return a / (1.0f + expf(-a)); }

// MODE 0: GEMM1 + SwiGLU -> bf16 h. MODE 1: GEMM2 -> fp32 y.
// SAVE_AB (MODE 0, training): the epilogue also keeps the pre-activations
// a = x.W1 and b = x.W3, rounded to bf16, as ab[row] = [a | b] for the
// backward pass (which then never recomputes GEMM1).
// GATHER (MODE 0 only): the A operand is pulled straight from the token
// activations x by the schedule Phi ("zero-copy, direct landing"), so no
// gathered copy of the tokens is materialised. Warps 0 and 3 (64 threads)
// copy the CTA's 128 A rows per K step with 16-byte cp.async: thread t owns
// the 16-byte chunk t % 8 of rows t / 8 + 8i (i < 16), written where the
// 128-byte swizzle puts it (chunk c of row r at c ^ (r % 8)); padding rows
// are zero-filled. A thread signals a stage once its copies into it have
// completed (cp.async groups, three stages behind) and it has fenced them to
// the async proxy that tcgen05.mma reads through; then one arrive per warp
// on the leader's full barrier. B still comes by TMA (warp 0, lane 0).
// CG = 1: one CTA per 128x256 tile. CG = 2: a cluster of two CTAs (a tcgen05
// CTA pair) per 256x256 tile; CTA r loads rows [128r, 128r+128) of A and
// columns [128r, 128r+128) of B, the leader (r = 0) issues the pair MMAs and
// each CTA drains its own 128 TMEM lanes.
// LAND (MODE 0, CG 2): the pull dispatch runs inside this kernel. Warp 3 of
// every CTA takes 128-row blocks of the expert-sorted layout in order from a
// device counter, copies each row from x through Phi into xg (16-byte loads
// and stores; padding rows zero-filled), and publishes the block with a
// release store of its flag. The TMA producer waits (bounded) for the flag of
// its CTA's 128 rows before it loads a tile's A operand, then issues a
// cross-proxy fence, since the rows were written through the generic proxy
// and TMA reads through the async proxy. Blocks are landed in the order the
// tiles are handed out, so the copies run ahead of the tensor cores and the
// HBM-bound gather overlaps the MMAs; no warp that lands rows ever waits.
// NARROW (with LAND): rows of at most 512 values, landed several per round
// (a separate instantiation, so the kernel for wider rows is unchanged).
template <int MODE, int CG, bool GATHER, bool SAVE_AB, bool LAND = false, bool NARROW = false>
__global__ void __launch_bounds__(kNumThreads, 1)
    ffn_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                    const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ CUtensorMap tmY,
                    const FfnParams p) {
  using C = Cfg<CG, MODE>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* staging = smem + C::STAGES * C::STAGE_BYTES;  // TMA_STORE only
  uint64_t* bars = reinterpret_cast<uint64_t*>(staging + C::STAGING_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NUM_BARS);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  int* bad_flag = abort_flag + 1;
  int* tile_ring = reinterpret_cast<int*>(tmem_slot + 4);       // [kRing] tile ids
  int32_t* s_off = reinterpret_cast<int32_t*>(tile_ring + kRing);  // [E+1] segment starts
  int32_t* s_end = s_off + (p.E + 1);                            // [E] end of real rows

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int E = p.E;
  const uint32_t rank = (CG == 2) ? cluster_ctarank() : 0u;
  const bool leader = rank == 0;

  if (tid == 0) {
    for (int i = 0; i < C::STAGES; ++i) {
      // GATHER: + one arrive per A-producer warp of each CTA of the pair
      mbar_init(smem_u32(&bars[C::BAR_FULL + i]), GATHER ? 1 + 2 * CG : 1);
      mbar_init(smem_u32(&bars[C::BAR_EMPTY + i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&bars[C::BAR_TFULL + i]), 1);
      mbar_init(smem_u32(&bars[C::BAR_TEMPTY + i]), kNumEpiWarps * CG);
    }
    mbar_init(smem_u32(&bars[C::BAR_DRAIN]), 1);
    for (int i = 0; i < kRing; ++i) {
      mbar_init(smem_u32(&bars[C::BAR_TID_FULL + i]), 1);
      // GATHER: warp 3 of each CTA reads the tile ids too
      mbar_init(smem_u32(&bars[C::BAR_TID_EMPTY + i]), C::TID_CONSUMERS + (GATHER ? CG : 0));
    }
    *abort_flag = 0;
    *bad_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB0);
    tma_prefetch_desc(&tmB1);
    if (C::TMA_STORE) tma_prefetch_desc(&tmY);
  }
  load_segments(p.offsets, p.counts, E, p.P, C::BM, p.rows_max, s_off, s_end, bad_flag);
  if (warp == 1) {
    if (CG == 2) {
      tmem_alloc_pair(smem_u32(tmem_slot), kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(tmem_slot), kTmemCols);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (CG == 2) cluster_sync();  // the peer's barriers exist before anything targets them
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const bool bad_sched = *bad_flag != 0;
  if (bad_sched && tid == 0) atomicOr(p.dev_status, MOE_DEV_BAD_SCHEDULE);

  const int rows_used = bad_sched ? 0 : s_off[E];
  const int tiles_n = (MODE == 0) ? p.Nout / 128 : p.Nout / C::BN;
  const int num_tiles = (rows_used / C::BM) * tiles_n;
  const int kblocks = p.K / C::BK;
  const WaitCtx wc{abort_flag, p.dev_status, p.timeout_ns, MOE_DEV_TIMEOUT};

  // Tiles come from the tile-id ring (persistent_gemm.cuh), filled by the
  // leader's scheduler thread from a device-wide counter.
  const uint32_t tid_empty_local = smem_u32(&bars[C::BAR_TID_EMPTY]);
  const TileRing tring{tile_ring, smem_u32(&bars[C::BAR_TID_FULL]), tid_empty_local,
                       (CG == 2) ? mapa_shared(tid_empty_local, 0) : tid_empty_local, !leader};
  auto next_tile = [&](int& pos, uint32_t& ph) -> int {
    return tring.next<CG == 2>(pos, ph, wc);
  };
  const int64_t drain_ns = p.timeout_ns < 100000000ll ? p.timeout_ns : 100000000ll;

  // tile -> (first row, n-tile, expert); false if the tile holds only padding.
  // Expert by expert, N-block-major inside chunks of RM M-tiles (RN = 1): each
  // weight column block's M-tiles run back to back and the chunk's A rows stay
  // in L2. With the dynamic tile order the tiles in flight are a narrow window
  // of ids, and this order measured faster for both GEMMs (GEMM1 21.8 vs
  // 22.7 ms against M-tile-major; GEMM2's DRAM reads equal W2 + h).
  auto tile_info = [&](int tile, int& row0, int& n, int& l) -> bool {
    return grouped_row_tile<C::BM, 8, 1>(tile, s_off, s_end, E, tiles_n, row0, n, l);
  };

  if ((warp == 0 || warp == 3) && GATHER) {
    // ------------------------------------------------------------ producers (row gather)
    constexpr int kLag = 3;  // cp.async groups in flight per thread before a stage is signalled
    static_assert(kLag < C::STAGES, "a stage is signalled before its slot is needed again");
    const int pt = (warp == 0 ? 0 : 32) + lane;  // producer thread 0..63
    const int cchunk = pt & 7;                   // 16-byte chunk of the 128-byte row
    const int r0 = pt >> 3;                      // rows r0 + 8i of the CTA's 128
    const uint32_t swz = static_cast<uint32_t>((cchunk ^ (r0 & 7)) << 4);
    const uint32_t full0 = smem_u32(&bars[C::BAR_FULL]);
    const uint32_t full_tgt0 = (CG == 2) ? mapa_shared(full0, 0) : full0;
    const uint16_t* xsrc = reinterpret_cast<const uint16_t*>(p.x);
    int stage = 0;
    uint32_t phase = 0;
    int64_t issued = 0, signalled = 0;
    bool ok = true;
    int bad = 0;
    int tpos = 0;
    uint32_t tph = 0;
    // make the copies of the oldest unsignalled stage visible to the async
    // proxy and arrive on its full barrier (once per warp)
    auto signal_oldest = [&](int keep) {
      if (keep == 0) asm volatile("cp.async.wait_group 0;" ::: "memory");
      else asm volatile("cp.async.wait_group %0;" ::"n"(kLag) : "memory");
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        const int st = static_cast<int>(signalled % C::STAGES);
        if (CG == 2 && !leader) mbar_arrive_cluster(full_tgt0 + st * 8);
        else mbar_arrive(full0 + st * 8);
      }
      ++signalled;
    };
    while (ok) {
      int tile = 0;
      if (lane == 0) tile = next_tile(tpos, tph);
      tile = __shfl_sync(0xFFFFFFFFu, tile, 0);
      if (tile < 0) break;
      int row0, n, l;
      if (!tile_info(tile, row0, n, l)) continue;
      const int arow = row0 + static_cast<int>(rank) * 128;
      // token rows of this thread's 16 A rows (padding and invalid entries: zero-fill)
      const uint16_t* src[16];
      uint32_t valid = 0;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int2 e = __ldg(p.phi + arow + r0 + 8 * i);
        const bool v = e.x >= 0 && e.x < p.P && e.y >= 0 && e.y < p.n_per_peer;
        if (!v && (e.x >= 0 || e.y != -1)) bad = 1;  // (-1,-1) is padding
        src[i] = xsrc + (v ? (static_cast<int64_t>(e.x) * p.n_per_peer + e.y) * p.K : 0) + cchunk * 8;
        valid |= (v ? 1u : 0u) << i;
      }
      const int ky0 = l * p.K;
      for (int kb = 0; kb < kblocks; ++kb) {
        uint32_t w_ok = 1;
        if (lane == 0) w_ok = wait_bounded(smem_u32(&bars[C::BAR_EMPTY + stage]), phase ^ 1u, wc) ? 1u : 0u;
        w_ok = __shfl_sync(0xFFFFFFFFu, w_ok, 0);
        if (!w_ok) {
          ok = false;
          break;
        }
        const uint32_t sA = smem_u32(smem + stage * C::STAGE_BYTES);
        const uint32_t sB = sA + C::A_BYTES;
        if (warp == 0 && lane == 0) {
          const uint32_t full_tgt = full_tgt0 + stage * 8;
          const int ky = ky0 + kb * C::BK;
          if (leader) mbar_arrive_expect_tx(full0 + stage * 8, CG * (C::STAGE_BYTES - C::A_BYTES));
          if (CG == 1) {
            tma_load_2d(sB + 0 * C::B_ATOM_BYTES, &tmB0, n * 128, ky, full_tgt);
            tma_load_2d(sB + 1 * C::B_ATOM_BYTES, &tmB0, n * 128 + 64, ky, full_tgt);
            tma_load_2d(sB + 2 * C::B_ATOM_BYTES, &tmB1, n * 128, ky, full_tgt);
            tma_load_2d(sB + 3 * C::B_ATOM_BYTES, &tmB1, n * 128 + 64, ky, full_tgt);
          } else {
            const CUtensorMap* mb = (rank == 1) ? &tmB1 : &tmB0;
            tma_load_2d_pair(sB, mb, n * 128, ky, full_tgt);
            tma_load_2d_pair(sB + C::B_ATOM_BYTES, mb, n * 128 + 64, ky, full_tgt);
          }
        }
        const int koff = kb * C::BK;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const uint32_t dst = sA + static_cast<uint32_t>((r0 + 8 * i) * 128) + swz;
          const uint32_t nbytes = ((valid >> i) & 1u) ? 16u : 0u;  // 0: zero-fill
          asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst),
                       "l"(src[i] + koff), "r"(nbytes)
                       : "memory");
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
        ++issued;
        if (++stage == C::STAGES) {
          stage = 0;
          phase ^= 1u;
        }
        if (issued - signalled > kLag) signal_oldest(kLag);
      }
    }
    if (ok) {
      while (signalled < issued) signal_oldest(0);
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");  // no copy may land after exit
    }
    if (bad) atomicOr(p.dev_status, MOE_DEV_BAD_SCHEDULE);
    __syncwarp();
    if (warp == 0 && lane == 0) {
      // no TMA load may still be landing in shared memory when the CTA exits
      const int64_t first = issued > C::STAGES ? issued - C::STAGES : 0;
      for (int64_t j = first; j < issued; ++j) {
        const int st = static_cast<int>(j % C::STAGES);
        const uint32_t par = static_cast<uint32_t>((j / C::STAGES) & 1);
        wait_drain(smem_u32(&bars[(leader ? C::BAR_FULL : C::BAR_EMPTY) + st]), par, drain_ns);
      }
    }
  } else if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      // the leader's full barriers count the bytes of both CTAs of a pair
      const uint32_t full0 = smem_u32(&bars[C::BAR_FULL]);
      const uint32_t full_tgt0 = (CG == 2) ? mapa_shared(full0, 0) : full0;
      int stage = 0;
      uint32_t phase = 0;
      int64_t issued = 0;
      bool ok = true;
      int tpos = 0;
      uint32_t tph = 0;
      while (ok) {
        const int tile = next_tile(tpos, tph);
        if (tile < 0) break;
        int row0, n, l;
        if (!tile_info(tile, row0, n, l)) continue;
        const int arow = row0 + static_cast<int>(rank) * 128;
        const int yb = l * p.K;
        if (LAND) {  // this CTA's 128 A rows must have landed
          if (!wait_flag_bounded(p.land_ready + arow / 128, wc)) break;
          asm volatile("fence.proxy.async.global;" ::: "memory");
        }
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!wait_bounded(smem_u32(&bars[C::BAR_EMPTY + stage]), phase ^ 1u, wc)) {
            ok = false;
            break;
          }
          const uint32_t full_local = full0 + stage * 8;
          const uint32_t full_tgt = full_tgt0 + stage * 8;
          const uint32_t sA = smem_u32(smem + stage * C::STAGE_BYTES);
          const uint32_t sB = sA + C::A_BYTES;
          const int ky = yb + kb * C::BK;
          if (leader) mbar_arrive_expect_tx(full_local, CG * C::STAGE_BYTES);
          if (CG == 1) {
            tma_load_2d(sA, &tmA, kb * C::BK, arow, full_tgt);
            if (MODE == 0) {
              tma_load_2d(sB + 0 * C::B_ATOM_BYTES, &tmB0, n * 128, ky, full_tgt);
              tma_load_2d(sB + 1 * C::B_ATOM_BYTES, &tmB0, n * 128 + 64, ky, full_tgt);
              tma_load_2d(sB + 2 * C::B_ATOM_BYTES, &tmB1, n * 128, ky, full_tgt);
              tma_load_2d(sB + 3 * C::B_ATOM_BYTES, &tmB1, n * 128 + 64, ky, full_tgt);
            } else {
#pragma unroll
              for (int b = 0; b < 4; ++b)
                tma_load_2d(sB + b * C::B_ATOM_BYTES, &tmB0, n * C::BN + b * 64, ky, full_tgt);
            }
          } else {
            tma_load_2d_pair(sA, &tmA, kb * C::BK, arow, full_tgt);
            // GEMM1: CTA 0 holds W1's columns, CTA 1 W3's (the two SwiGLU halves);
            // GEMM2: CTA r holds W2 columns [n*256 + 128r, +128).
            const CUtensorMap* mb = (MODE == 0 && rank == 1) ? &tmB1 : &tmB0;
            const int x0 = (MODE == 0) ? n * 128 : n * C::BN + static_cast<int>(rank) * 128;
            tma_load_2d_pair(sB, mb, x0, ky, full_tgt);
            tma_load_2d_pair(sB + C::B_ATOM_BYTES, mb, x0 + 64, ky, full_tgt);
          }
          ++issued;
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // no load may still be landing in shared memory when the CTA exits: the
      // leader sees its full barriers complete; a follower sees the stage
      // released by the leader's MMAs (which waited for the data)
      const int64_t first = issued > C::STAGES ? issued - C::STAGES : 0;
      for (int64_t j = first; j < issued; ++j) {
        const int st = static_cast<int>(j % C::STAGES);
        const uint32_t par = static_cast<uint32_t>((j / C::STAGES) & 1);
        wait_drain(smem_u32(&bars[(leader ? C::BAR_FULL : C::BAR_EMPTY) + st]), par, drain_ns);
      }
    }
  } else if (warp == 3 && LAND) {
    // ------------------------------------------------------------ pull dispatch
    const int nblk = rows_used / 128;
    const int chunks = p.K / 8;  // 16-byte chunks per row (H % 256 == 0: a multiple of 32)
    const uint4* xsrc = reinterpret_cast<const uint4*>(p.x);
    int bad = 0;
    for (;;) {
      int b = 0;
      if (lane == 0) b = atomicAdd(p.land_next, 1);
      b = __shfl_sync(0xFFFFFFFFu, b, 0);
      if (b >= nblk || *wc.abort) break;
      constexpr int U = 28;  // 16-byte loads in flight per lane: a 7,168-wide row in one round
      constexpr int UR = 16;  // the same for rows of at most 512 values, several per round
      if (NARROW) {
        // narrow rows (one or two loads per lane), whole rows per round: lane
        // j takes chunks j, j+32, ... of the round's rows back to back
        // (chunks is a multiple of 32), so the rows share a round instead of
        // each costing a memory round trip
        const int rpr = (32 * UR) / chunks;  // 8 or 16
#pragma unroll 1
        for (int rr0 = 0; rr0 < 128; rr0 += rpr) {
          // lane l < rpr looks up row rr0 + l once: the chunk offset of its
          // token row, -1 for padding; each load below takes its row's by shuffle
          int64_t so_l = -1;
          if (lane < rpr && rr0 + lane < 128) {
            const int2 e = __ldg(p.phi + static_cast<int64_t>(b) * 128 + rr0 + lane);
            const bool v = e.x >= 0 && e.x < p.P && e.y >= 0 && e.y < p.n_per_peer;
            if (!v && (e.x >= 0 || e.y != -1)) bad = 1;  // (-1,-1) is padding
            if (v) so_l = (static_cast<int64_t>(e.x) * p.n_per_peer + e.y) * chunks;
          }
          uint4 t[UR];
          int ro = 0, c = lane;
#pragma unroll
          for (int u = 0; u < UR; ++u) {
            const int64_t so = __shfl_sync(0xFFFFFFFFu, so_l, ro);
            t[u] = (ro < rpr && so >= 0) ? __ldg(xsrc + so + c) : make_uint4(0, 0, 0, 0);
            c += 32;
            if (c >= chunks) {
              c -= chunks;
              ++ro;
            }
          }
          ro = 0;
          c = lane;
#pragma unroll
          for (int u = 0; u < UR; ++u) {
            const int rr = rr0 + ro;
            if (ro < rpr && rr < 128)
              reinterpret_cast<uint4*>(p.xg)[(static_cast<int64_t>(b) * 128 + rr) * chunks + c] =
                  t[u];
            c += 32;
            if (c >= chunks) {
              c -= chunks;
              ++ro;
            }
          }
        }
      } else {
#pragma unroll 1
        for (int rr = 0; rr < 128; ++rr) {
          const int64_t row = static_cast<int64_t>(b) * 128 + rr;
          const int2 e = __ldg(p.phi + row);
          const bool v = e.x >= 0 && e.x < p.P && e.y >= 0 && e.y < p.n_per_peer;
          if (!v && (e.x >= 0 || e.y != -1)) bad = 1;  // (-1,-1) is padding
          uint4* dst = reinterpret_cast<uint4*>(p.xg) + row * chunks;
          const uint4* src =
              xsrc + (v ? (static_cast<int64_t>(e.x) * p.n_per_peer + e.y) * chunks : 0);
#pragma unroll 1
          for (int c0 = lane; c0 < chunks; c0 += 32 * U) {
            uint4 t[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
              const int c = c0 + 32 * u;
              t[u] = (v && c < chunks) ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
              const int c = c0 + 32 * u;
              if (c < chunks) dst[c] = t[u];
            }
          }
        }
      }
      __threadfence();  // every lane's rows before the flag
      __syncwarp();
      if (lane == 0)
        asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p.land_ready + b), "r"(1)
                     : "memory");
    }
    if (bad) atomicOr(p.dev_status, MOE_DEV_BAD_SCHEDULE);
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && leader) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      int tpos = 0;
      uint32_t tph = 0;
      while (ok) {
        const int tile = next_tile(tpos, tph);
        if (tile < 0) break;
        int row0, n, l;
        if (!tile_info(tile, row0, n, l)) continue;
        if (!wait_bounded<CG == 2>(smem_u32(&bars[C::BAR_TEMPTY + acc]), acc_phase ^ 1u, wc)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * C::BN);
        for (int kb = 0; kb < kblocks; ++kb) {
          // GATHER with CTA pairs: the follower's producers release its A rows
          // at cluster scope, so the wait acquires at cluster scope
          if (!wait_bounded<GATHER && CG == 2>(smem_u32(&bars[C::BAR_FULL + stage]), phase, wc)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sA = smem_u32(smem + stage * C::STAGE_BYTES);
          const uint32_t sB = sA + C::A_BYTES;
#pragma unroll
          for (int kk = 0; kk < C::BK / kUmmaK; ++kk) {
            // A: K-major, advance 16 bf16 = 32 bytes inside the swizzled row.
            // B: MN-major, advance 16 K-rows = two 8-row groups = 2048 bytes.
            const uint64_t a_desc = smem_desc_sw128(sA + kk * 32, 16, 1024);
            const uint64_t b_desc = smem_desc_sw128(sB + kk * 2048, C::B_ATOM_BYTES, 1024);
            const uint32_t accum = (kb | kk) != 0 ? 1u : 0u;
            if (CG == 2) tc_mma_f16_pair(d_tmem, a_desc, b_desc, C::IDESC, accum);
            else tc_mma_f16(d_tmem, a_desc, b_desc, C::IDESC, accum);
          }
          if (CG == 2) tc_commit_pair_mc(smem_u32(&bars[C::BAR_EMPTY + stage]), 0x3);
          else tc_commit(smem_u32(&bars[C::BAR_EMPTY + stage]));
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        if (CG == 2) tc_commit_pair_mc(smem_u32(&bars[C::BAR_TFULL + acc]), 0x3);
        else tc_commit(smem_u32(&bars[C::BAR_TFULL + acc]));
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      // all MMAs issued by this thread have completed once this arrives
      if (CG == 2) tc_commit_pair(smem_u32(&bars[C::BAR_DRAIN]));
      else tc_commit(smem_u32(&bars[C::BAR_DRAIN]));
      wait_drain(smem_u32(&bars[C::BAR_DRAIN]), 0, p.timeout_ns);
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ tile scheduler
    if (lane == 0 && leader) tring.schedule<CG == 2>(p.tile_counter, num_tiles, wc);
  } else if (warp >= kEpiWarp0) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                  // TMEM lane quarter this warp may access
    const int half = (warp - kEpiWarp0) >> 2;  // which half of the tile's columns
    const uint32_t tempty0 = smem_u32(&bars[C::BAR_TEMPTY]);
    const uint32_t tempty_tgt0 = (CG == 2) ? mapa_shared(tempty0, 0) : tempty0;
    int acc = 0;
    uint32_t acc_phase = 0;
    int tpos = 0;
    uint32_t tph = 0;
    for (;;) {
      int tile = 0;
      if (lane == 0) tile = next_tile(tpos, tph);
      tile = __shfl_sync(0xFFFFFFFFu, tile, 0);
      if (tile < 0) break;
      int row0, n, l;
      if (!tile_info(tile, row0, n, l)) continue;
      if (!wait_bounded(smem_u32(&bars[C::BAR_TFULL + acc]), acc_phase, wc)) break;
      tc_fence_after();
      const int64_t row = row0 + static_cast<int>(rank) * 128 + q * 32 + lane;
      const uint32_t tbase =
          tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * C::BN);
      // TMEM reads are double-buffered: chunk c+1 is in flight while chunk c
      // is converted and stored.
      if (MODE == 0) {
        // accumulator columns [0,128) = x.W1, [128,256) = x.W3 for h columns n*128 + j
        __nv_bfloat16* hrow =
            reinterpret_cast<__nv_bfloat16*>(p.out) + row * p.Nout + n * 128 + half * 64;
        uint32_t ra[2][32], rb[2][32];
        tmem_ld_32cols(tbase + half * 64, ra[0]);
        tmem_ld_32cols(tbase + 128 + half * 64, rb[0]);
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          if (c + 1 < 2) {
            tmem_ld_32cols(tbase + half * 64 + (c + 1) * 32, ra[(c + 1) & 1]);
            tmem_ld_32cols(tbase + 128 + half * 64 + (c + 1) * 32, rb[(c + 1) & 1]);
          }
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float h0 = silu(__uint_as_float(ra[c & 1][2 * i])) * __uint_as_float(rb[c & 1][2 * i]);
            const float h1 =
                silu(__uint_as_float(ra[c & 1][2 * i + 1])) * __uint_as_float(rb[c & 1][2 * i + 1]);
            pk[i] = pack_bf16x2(h0, h1);
          }
          st_global_v8(hrow + c * 32, *reinterpret_cast<const uint32_t(*)[8]>(&pk[0]));
          st_global_v8(hrow + c * 32 + 16, *reinterpret_cast<const uint32_t(*)[8]>(&pk[8]));
          if (SAVE_AB) {
            __nv_bfloat16* arow = reinterpret_cast<__nv_bfloat16*>(p.ab) + row * (2 * p.Nout) +
                                  n * 128 + half * 64 + c * 32;
            __nv_bfloat16* brow = arow + p.Nout;
#pragma unroll
            for (int v = 0; v < 2; ++v) {
              uint32_t qa[8], qb[8];
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                qa[i] = pack_bf16x2(__uint_as_float(ra[c & 1][16 * v + 2 * i]),
                                    __uint_as_float(ra[c & 1][16 * v + 2 * i + 1]));
                qb[i] = pack_bf16x2(__uint_as_float(rb[c & 1][16 * v + 2 * i]),
                                    __uint_as_float(rb[c & 1][16 * v + 2 * i + 1]));
              }
              st_global_v8(arow + 16 * v, qa);
              st_global_v8(brow + 16 * v, qb);
            }
          }
          if (c + 1 < 2) tmem_ld_wait();
        }
      } else if (C::TMA_STORE) {
        // row `lane` of this warp's 32x16 block goes to the staging slot with
        // 16-byte chunk j at position j ^ ((lane >> 1) & 3): the 64-byte swizzle
        // the tensor map expects, and no bank conflicts for the 16-byte writes.
        const uint32_t stg = smem_u32(staging) + (warp - kEpiWarp0) * 2048;
        const uint64_t pol_y = l2_policy_evict_first();
        const int ycol = n * C::BN + half * 128;
        const int yrow0 = row0 + static_cast<int>(rank) * 128 + q * 32;
        // a 32-row block wholly past the expert's routes holds only padding
        // rows, which nothing reads: its y is not written
        const bool keep = yrow0 < s_end[l];
        uint32_t rv[2][16];
        tmem_ld_16cols(tbase + half * 128, rv[0]);
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          if (c + 1 < 8) tmem_ld_16cols(tbase + half * 128 + (c + 1) * 16, rv[(c + 1) & 1]);
          if (keep) {
            if (lane == 0) bulk_wait_read_all();  // the previous store has read the slot
            __syncwarp();
#pragma unroll
            for (int j = 0; j < 4; ++j)
              st_shared_v4(stg + lane * 64 + ((j ^ ((lane >> 1) & 3)) << 4), rv[c & 1][4 * j],
                           rv[c & 1][4 * j + 1], rv[c & 1][4 * j + 2], rv[c & 1][4 * j + 3]);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {  // y is streamed out and read once, by the combine
              tma_store_2d_hint(&tmY, stg, ycol + c * 16, yrow0, pol_y);
              bulk_commit_group();
            }
          }
          if (c + 1 < 8) tmem_ld_wait();
        }
      } else {
        float* yrow = reinterpret_cast<float*>(p.out) + row * p.Nout + n * C::BN + half * 128;
        uint32_t rv[2][32];
        tmem_ld_32cols(tbase + half * 128, rv[0]);
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          if (c + 1 < 4) tmem_ld_32cols(tbase + half * 128 + (c + 1) * 32, rv[(c + 1) & 1]);
#pragma unroll
          for (int v = 0; v < 4; ++v)
            st_global_v8(yrow + c * 32 + v * 8,
                         *reinterpret_cast<const uint32_t(*)[8]>(&rv[c & 1][8 * v]));
          if (c + 1 < 4) tmem_ld_wait();
        }
      }
      // The accumulator may be overwritten once every lane's tcgen05.ld has
      // completed (tcgen05.wait::ld above); the global stores need no ordering
      // against the next MMAs, so the arrive is relaxed (no memory fence).
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (CG == 2) mbar_arrive_relaxed_cluster(tempty_tgt0 + acc * 8);
        else mbar_arrive_relaxed(tempty0 + acc * 8);
      }
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
    if (C::TMA_STORE && lane == 0) bulk_wait_all();  // stores complete before the CTA exits
  }

  __syncthreads();
  if (CG == 2) cluster_sync();  // the peer no longer reads this CTA's smem or TMEM
  if (tid == 0) finish_tile_counter(p.tile_counter);
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    if (CG == 2) tmem_dealloc_pair(tmem_base, kTmemCols);
    else tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace

namespace {

template <int MODE, int CG, bool GATHER = false, bool SAVE_AB = false, bool LAND = false,
          bool NARROW = false>
cudaError_t launch_mode(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                        const CUtensorMap& yo, FfnParams p, cudaStream_t s) {
  const size_t smem = smem_bytes_for<CG, MODE>(p.E);
  if (!p.tile_counter) {  // no counter of the caller's: one from the device's pool
    const cudaError_t e = tile_counter_for_current_device(&p.tile_counter);
    if (e != cudaSuccess) return e;
  }
  return launch_persistent(ffn_gemm_kernel<MODE, CG, GATHER, SAVE_AB, LAND, NARROW>, CG, smem, s,
                           a, b0, b1, yo, p);
}

}  // namespace

cudaError_t launch_expert_ffn(const uint16_t* xg, const uint16_t* W1, const uint16_t* W3,
                              const uint16_t* W2, const int32_t* offsets, const int32_t* counts,
                              uint16_t* h, float* y, const moe_shape_t& sh, int64_t rows_max,
                              int32_t* dev_status, cudaStream_t s, cudaEvent_t ev_mid,
                              uint16_t* ab, int* counter, const LandArgs* land) {
  const int E = sh.E, H = sh.H, I = sh.I;
  CUtensorMap mA1, mW1, mW3, mA2, mW2, mY;
  const uint64_t EH = static_cast<uint64_t>(E) * H, EI = static_cast<uint64_t>(E) * I;
  if (!make_map(&mA1, xg, H, rows_max, 64, 128) || !make_map(&mW1, W1, I, EH, 64, 64) ||
      !make_map(&mW3, W3, I, EH, 64, 64) || !make_map(&mA2, h, I, rows_max, 64, 128) ||
      !make_map(&mW2, W2, H, EI, 64, 64) || !make_map(&mY, y, H, rows_max, 16, 32, true, true))
    return cudaErrorInvalidValue;
  // Segments that are multiples of 256 rows run on CTA pairs (256x256 tiles);
  // otherwise (pad a multiple of 128 only) on single CTAs (128x256 tiles).
  const bool pair = (sh.pad % 256) == 0;
  FfnParams p1{counter, nullptr, 0, offsets, counts, E, sh.P, H, I, rows_max, h, dev_status,
               kWaitTimeoutNs, ab};
  cudaError_t e;
  if (land) {  // the pull dispatch fused into GEMM1 (pair tiles only)
    if (!pair) return cudaErrorInvalidValue;
    p1.phi = reinterpret_cast<const int2*>(land->phi);
    p1.n_per_peer = sh.N;
    p1.x = land->x;
    p1.xg = const_cast<uint16_t*>(xg);
    p1.land_next = land->next;
    p1.land_ready = land->ready;
    if (H <= 512)  // rows of one or two 16-byte chunks per lane: several per round
      e = ab ? launch_mode<0, 2, false, true, true, true>(mA1, mW1, mW3, mA1, p1, s)
             : launch_mode<0, 2, false, false, true, true>(mA1, mW1, mW3, mA1, p1, s);
    else
      e = ab ? launch_mode<0, 2, false, true, true>(mA1, mW1, mW3, mA1, p1, s)
             : launch_mode<0, 2, false, false, true>(mA1, mW1, mW3, mA1, p1, s);
  } else if (ab) {  // training: keep the pre-activations (pair tiles only)
    e = pair ? launch_mode<0, 2, false, true>(mA1, mW1, mW3, mA1, p1, s) : cudaErrorInvalidValue;
  } else {
    e = pair ? launch_mode<0, 2>(mA1, mW1, mW3, mA1, p1, s) : launch_mode<0, 1>(mA1, mW1, mW3, mA1, p1, s);
  }
  if (e != cudaSuccess) return e;
  if (ev_mid) {
    e = cudaEventRecord(ev_mid, s);
    if (e != cudaSuccess) return e;
  }
  FfnParams p2{counter, nullptr, 0, offsets, counts, E, sh.P, I, H, rows_max, y, dev_status,
               kWaitTimeoutNs, nullptr};
  return pair ? launch_mode<1, 2>(mA2, mW2, mW2, mY, p2, s)
              : launch_mode<1, 1>(mA2, mW2, mW2, mY, p2, s);
}

cudaError_t launch_expert_ffn_gather(const uint16_t* x, const int32_t* phi, const uint16_t* W1,
                                     const uint16_t* W3, const uint16_t* W2,
                                     const int32_t* offsets, const int32_t* counts, uint16_t* h,
                                     float* y, const moe_shape_t& sh, int64_t rows_max,
                                     int32_t* dev_status, cudaStream_t s, cudaEvent_t ev_mid) {
  const int E = sh.E, H = sh.H, I = sh.I;
  CUtensorMap mW1, mW3, mA2, mW2, mY;
  const uint64_t EH = static_cast<uint64_t>(E) * H, EI = static_cast<uint64_t>(E) * I;
  if (!make_map(&mW1, W1, I, EH, 64, 64) || !make_map(&mW3, W3, I, EH, 64, 64) ||
      !make_map(&mA2, h, I, rows_max, 64, 128) || !make_map(&mW2, W2, H, EI, 64, 64) ||
      !make_map(&mY, y, H, rows_max, 16, 32, true, true))
    return cudaErrorInvalidValue;
  const bool pair = (sh.pad % 256) == 0;
  // GEMM1's A rows come from x by Phi (cp.async); its A tensor map is unused
  FfnParams p1{nullptr, reinterpret_cast<const int2*>(phi), sh.N, offsets, counts, E, sh.P, H,
               I, rows_max, h, dev_status, kWaitTimeoutNs, nullptr, x};
  cudaError_t e = pair ? launch_mode<0, 2, true>(mW1, mW1, mW3, mW1, p1, s)
                       : launch_mode<0, 1, true>(mW1, mW1, mW3, mW1, p1, s);
  if (e != cudaSuccess) return e;
  if (ev_mid) {
    e = cudaEventRecord(ev_mid, s);
    if (e != cudaSuccess) return e;
  }
  FfnParams p2{nullptr, nullptr, 0, offsets, counts, E, sh.P, I, H, rows_max, y, dev_status,
               kWaitTimeoutNs, nullptr, nullptr};
  return pair ? launch_mode<1, 2>(mA2, mW2, mW2, mY, p2, s)
              : launch_mode<1, 1>(mA2, mW2, mW2, mY, p2, s);
}

// ---------------------------------------------------------------- self test
namespace {
__global__ void selftest_wait_kernel(int32_t* dev_status, int64_t timeout_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const WaitCtx wc{&abort_flag, dev_status, timeout_ns, MOE_DEV_TIMEOUT};
    // phase 0 never completes: nothing arrives on this barrier
    wait_bounded(smem_u32(&bar), 0, wc);
  }
}
}  // namespace

cudaError_t launch_selftest_wait(int32_t* dev_status, int64_t timeout_ns, cudaStream_t s) {
  selftest_wait_kernel<<<1, 32, 0, s>>>(dev_status, timeout_ns);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace moe
