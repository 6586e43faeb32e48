// Backward of the grouped SwiGLU expert FFN on the 5th-generation tensor cores.
//
// "Mixture-of-Kittens: A MoE Megakernel for GB300 NVL72": the one schedule
// table Phi serves the backward phases too (overview; section 2: backward =
// pull-reverse-combine, push-reverse-dispatch), weight gradients are deferred
// until every activation gradient is done and accumulated over the token
// dimension in one pass (overview, backward execution step), and the router
// gradient comes from the inner product of the SwiGLU activations with the
// down-projection dgrads, so the down projection's output is never kept
// (section 5, SonicMoE gradients).
//
// Per route row (token t, slot j, expert e, gate g; dys = dout[t]):
//   DGRAD_H  dhu = dys . W2[e]^T            (fp32 in TMEM; M = rows, N = I, K = H)
//            epilogue: dgate partial = sum h * dhu over the tile's columns,
//            dh = g * dhu, s = sigmoid(a),
//            da = dh * b * s * (1 + a * (1 - s)), db = dh * a * s, hg = g * h
//            (a, b: the forward's saved bf16 pre-activations; da, db, hg
//            stored as bf16: they are operands of the next GEMMs)
//   DGRAD_X  dxg = [da | db] . [W1[e] | W3[e]]^T   (M = rows, N = H, K = 2I) -> fp32
//   WGRAD    per expert, over the rows it received (K = rows):
//            dW2[e] = hg^T . dys   (M = I, N = H)
//            [dW1[e] | dW3[e]] = xg^T . [da | db]  (M = H, N = 2I)  -> fp32
//
// Design: the forward's persistent warp-specialised CTA-pair kernel (see
// expert_ffn.cu) with the operand majors each product needs. The dgrads read
// the weights as stored ([E, I, H] for W2, [E, H, I] for W1/W3) with K along
// the contiguous dimension: a K-major B operand, 128 rows x 64 K per CTA and
// stage. The wgrads reduce over rows, the outer dimension of both operands:
// A and B are MN-major (64-column atoms of 64 rows), exactly the layout the
// forward uses for its weight operand. Tiles are 256 x 256 on CTA pairs
// (tcgen05.mma.cta_group::2, M = 256, N = 256, K = 16 per instruction); the
// accumulator is double-buffered in TMEM. dxg leaves through 128-byte-
// swizzled staging and TMA stores (as the forward's y); the weight gradients
// leave with direct 32-byte stores: their tiles have short K (an expert's
// ~1,200 rows), and the staging chain (wait until the previous store has read
// the slot) then exposed its latency -- measured, dW2 12.8 vs 15.0 ms and
// dW1|dW3 25.0 vs 29.7 ms at the Kimi shape (the dxg GEMM, K = 2I, is faster
// with the TMA stores: 24.3 vs 27.2 ms).
//
// Determinism: every output element is produced by one CTA pair in a fixed K
// order (no split-K, no atomics). The gate gradient of a row is split over
// the I/128 column halves of its DGRAD_H tiles; the halves are written to
// separate slots and summed later in a fixed order (router backward).
//
// Weight gradients run over the expert's real rows rounded up to the K step
// of 64; the rows past the last route are padding rows of a computed tile,
// zero in every operand (the dispatch and the reverse combine write zero
// padding rows, the gates of padding rows are zero). An expert that received
// no route gets an all-zero gradient, written without any MMA.
#include <cuda_bf16.h>

#include "internal.cuh"
#include "persistent_gemm.cuh"
#include "sm100.cuh"

namespace moe {
namespace {

using namespace sm100;
using namespace pg;

enum : int { OP_DGRAD_H = 0, OP_DGRAD_X = 1, OP_WGRAD = 2 };

template <int OP>
struct BCfg {
  static constexpr bool WGRAD = OP == OP_WGRAD;
  static constexpr bool TMA_STORE = OP == OP_DGRAD_X;
  static constexpr int STAGING_BYTES = TMA_STORE ? 8 * 4096 : 0;  // 8 warps x 32x32 fp32
  static constexpr int BM = 256, BN = 256, BK = 64;
  static constexpr int A_BYTES = 128 * BK * 2;     // this CTA's 128 M x 64 K
  static constexpr int B_BYTES = 128 * BK * 2;     // this CTA's 128 N x 64 K
  static constexpr int ATOM_BYTES = 64 * BK * 2;   // MN-major: 64 columns x 64 K rows
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;  // 32 KB
  static constexpr int STAGES = TMA_STORE ? 5 : 6;
  static constexpr uint32_t IDESC = idesc_bf16_f32(BM, BN, WGRAD ? 1 : 0, WGRAD ? 1 : 0);
  static constexpr int BAR_FULL = 0;
  static constexpr int BAR_EMPTY = STAGES;
  static constexpr int BAR_TFULL = 2 * STAGES;
  static constexpr int BAR_TEMPTY = 2 * STAGES + 2;
  static constexpr int BAR_DRAIN = 2 * STAGES + 4;
  static constexpr int BAR_TID_FULL = 2 * STAGES + 5;
  static constexpr int BAR_TID_EMPTY = 2 * STAGES + 9;
  static constexpr int NUM_BARS = 2 * STAGES + 13;
  // readers of each tile id: producer, MMA issuer and 8 epilogue warps of the
  // leader; producer and 8 epilogue warps of the follower
  static constexpr int TID_CONSUMERS = 19;
  static_assert(STAGE_BYTES % 1024 == 0 && A_BYTES % 1024 == 0, "swizzle atoms stay 1024-aligned");
};

struct BwdParams {
  int* tile_counter;       // {next tile to hand out, CTAs finished}; zero at launch
  const int32_t* offsets;  // [E+1] segment starts
  const int32_t* counts;   // [E, P] routes per (expert, peer), or null (whole segments)
  int32_t E, P;
  int32_t K;        // dgrads: reduction length (H for DGRAD_H, 2I for DGRAD_X)
  int32_t kswitch;  // DGRAD_X: K index where the B operand moves from W1 to W3 (I)
  int32_t M;        // WGRAD: rows of each expert's gradient (I for dW2, H for dW1|dW3)
  int32_t N;        // output columns (I for DGRAD_H, H for DGRAD_X, H or 2I for WGRAD)
  int32_t nsplit;   // WGRAD: columns [0, nsplit) go to out0, the rest to out1
  int64_t rows_max;
  // DGRAD_H epilogue
  const uint16_t* ab;      // [rows_max, 2I] bf16 saved pre-activations a | b
  const uint16_t* h;       // [rows_max, I] bf16 forward SwiGLU output
  const float* gate_row;   // [rows_max] gate of each row's route (0 for padding)
  uint16_t* dab;           // [rows_max, 2I] bf16 da | db
  uint16_t* hg;            // [rows_max, I] bf16 g * h
  float* part;             // [rows_max, I/128] gate-gradient partial sums
  float* out0;             // WGRAD: output columns [0, nsplit)
  float* out1;             // WGRAD: output columns [nsplit, N)
  int32_t* dev_status;
  int64_t timeout_ns;
};

template <int OP>
size_t bwd_smem_bytes(int E) {
  using C = BCfg<OP>;
  return 1024 + static_cast<size_t>(C::STAGES) * C::STAGE_BYTES + C::STAGING_BYTES +
         C::NUM_BARS * 8 + 16 + kRing * 4 + static_cast<size_t>(2 * E + 1) * 4;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ void st_global_v4(void* ptr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.global.v4.b32 [%0], {%1, %2, %3, %4};" ::"l"(ptr), "r"(a), "r"(b), "r"(c), "r"(d)
               : "memory");
}

template <int OP>
__global__ void __launch_bounds__(kNumThreads, 1)
    ffn_bwd_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                   const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ CUtensorMap tmY0,
                   const __grid_constant__ CUtensorMap tmY1, const BwdParams p) {
  using C = BCfg<OP>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* staging = smem + C::STAGES * C::STAGE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(staging + C::STAGING_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NUM_BARS);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  int* bad_flag = abort_flag + 1;
  int* tile_ring = reinterpret_cast<int*>(tmem_slot + 4);
  int32_t* s_off = reinterpret_cast<int32_t*>(tile_ring + kRing);  // [E+1]
  int32_t* s_end = s_off + (p.E + 1);                            // [E] end of real rows

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int E = p.E;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;

  if (tid == 0) {
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(smem_u32(&bars[C::BAR_FULL + i]), 1);
      mbar_init(smem_u32(&bars[C::BAR_EMPTY + i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&bars[C::BAR_TFULL + i]), 1);
      mbar_init(smem_u32(&bars[C::BAR_TEMPTY + i]), kNumEpiWarps * 2);
    }
    mbar_init(smem_u32(&bars[C::BAR_DRAIN]), 1);
    for (int i = 0; i < kRing; ++i) {
      mbar_init(smem_u32(&bars[C::BAR_TID_FULL + i]), 1);
      mbar_init(smem_u32(&bars[C::BAR_TID_EMPTY + i]), C::TID_CONSUMERS);
    }
    *abort_flag = 0;
    *bad_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB0);
    tma_prefetch_desc(&tmB1);
    if (C::TMA_STORE) {
      tma_prefetch_desc(&tmY0);
      tma_prefetch_desc(&tmY1);
    }
  }
  load_segments(p.offsets, p.counts, E, p.P, C::BM, p.rows_max, s_off, s_end, bad_flag);
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the peer's barriers exist before anything targets them
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const bool bad_sched = *bad_flag != 0;
  if (bad_sched && tid == 0) atomicOr(p.dev_status, MOE_DEV_BAD_SCHEDULE);

  const int tiles_n = p.N / C::BN;
  const int tiles_m = C::WGRAD ? p.M / C::BM : 0;
  const int tiles_per_expert = tiles_m * tiles_n;
  const int num_tiles =
      bad_sched ? 0 : (C::WGRAD ? E * tiles_per_expert : (s_off[E] / C::BM) * tiles_n);
  const WaitCtx wc{abort_flag, p.dev_status, p.timeout_ns, MOE_DEV_TIMEOUT};

  // Tiles come from the tile-id ring (persistent_gemm.cuh), filled by the
  // leader's scheduler thread from a device-wide counter.
  const uint32_t tid_empty_local = smem_u32(&bars[C::BAR_TID_EMPTY]);
  const TileRing tring{tile_ring, smem_u32(&bars[C::BAR_TID_FULL]), tid_empty_local,
                       mapa_shared(tid_empty_local, 0), !leader};
  auto next_tile = [&](int& pos, uint32_t& ph) -> int { return tring.next<true>(pos, ph, wc); };
  const int64_t drain_ns = p.timeout_ns < 100000000ll ? p.timeout_ns : 100000000ll;

  // tile -> (first row, m-tile, n-tile, expert, K steps); false: skip (padding only).
  // dgrads: tiles are numbered expert by expert over the row tiles, in the
  // forward's grouped raster (N-block-major inside chunks of RM M-tiles).
  // WGRAD: expert-major, then m, then n.
  constexpr int RM = 8;
  constexpr int RN = 1;
  auto tile_info = [&](int tile, int& row0, int& m, int& n, int& l, int& kblocks) -> bool {
    if (C::WGRAD) {
      l = tile / tiles_per_expert;
      const int j = tile - l * tiles_per_expert;
      m = j / tiles_n;
      n = j - m * tiles_n;
      row0 = s_off[l];
      kblocks = (s_end[l] - s_off[l] + C::BK - 1) / C::BK;
      return true;
    }
    m = 0;
    kblocks = p.K / C::BK;
    return grouped_row_tile<C::BM, RM, RN>(tile, s_off, s_end, E, tiles_n, row0, n, l);
  };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint32_t full0 = smem_u32(&bars[C::BAR_FULL]);
      const uint32_t full_tgt0 = mapa_shared(full0, 0);
      int stage = 0;
      uint32_t phase = 0;
      int64_t issued = 0;
      bool ok = true;
      int tpos = 0;
      uint32_t tph = 0;
      while (ok) {
        const int tile = next_tile(tpos, tph);
        if (tile < 0) break;
        int row0, m, n, l, kblocks;
        if (!tile_info(tile, row0, m, n, l, kblocks)) continue;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!wait_bounded(smem_u32(&bars[C::BAR_EMPTY + stage]), phase ^ 1u, wc)) {
            ok = false;
            break;
          }
          const uint32_t full_local = full0 + stage * 8;
          const uint32_t full_tgt = full_tgt0 + stage * 8;
          const uint32_t sA = smem_u32(smem + stage * C::STAGE_BYTES);
          const uint32_t sB = sA + C::A_BYTES;
          if (leader) mbar_arrive_expect_tx(full_local, 2 * C::STAGE_BYTES);
          if (C::WGRAD) {
            // both operands MN-major: rows [row0 + 64 kb, +64) of the sources,
            // this CTA's 128 of the tile's M (resp. N) columns as two 64-column atoms
            const int ky = row0 + kb * C::BK;
            const int ax = m * C::BM + static_cast<int>(rank) * 128;
            const int bx = n * C::BN + static_cast<int>(rank) * 128;
            tma_load_2d_pair(sA, &tmA, ax, ky, full_tgt);
            tma_load_2d_pair(sA + C::ATOM_BYTES, &tmA, ax + 64, ky, full_tgt);
            tma_load_2d_pair(sB, &tmB0, bx, ky, full_tgt);
            tma_load_2d_pair(sB + C::ATOM_BYTES, &tmB0, bx + 64, ky, full_tgt);
          } else {
            // A: rows of the gathered operand, K-major. B: the expert's weight
            // rows n*256 + 128*rank .. +128 (output columns), K-major.
            const int kx = kb * C::BK;
            const bool second = (OP == OP_DGRAD_X) && kx >= p.kswitch;
            tma_load_2d_pair(sA, &tmA, kx, row0 + static_cast<int>(rank) * 128, full_tgt);
            tma_load_2d_pair(sB, second ? &tmB1 : &tmB0, second ? kx - p.kswitch : kx,
                             l * p.N + n * C::BN + static_cast<int>(rank) * 128, full_tgt);
          }
          ++issued;
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      const int64_t first = issued > C::STAGES ? issued - C::STAGES : 0;
      for (int64_t j = first; j < issued; ++j) {
        const int st = static_cast<int>(j % C::STAGES);
        const uint32_t par = static_cast<uint32_t>((j / C::STAGES) & 1);
        wait_drain(smem_u32(&bars[(leader ? C::BAR_FULL : C::BAR_EMPTY) + st]), par, drain_ns);
      }
    }
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
        int row0, m, n, l, kblocks;
        if (!tile_info(tile, row0, m, n, l, kblocks) || kblocks == 0) continue;
        if (!wait_bounded<true>(smem_u32(&bars[C::BAR_TEMPTY + acc]), acc_phase ^ 1u, wc)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * C::BN);
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!wait_bounded(smem_u32(&bars[C::BAR_FULL + stage]), phase, wc)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sA = smem_u32(smem + stage * C::STAGE_BYTES);
          const uint32_t sB = sA + C::A_BYTES;
#pragma unroll
          for (int kk = 0; kk < C::BK / kUmmaK; ++kk) {
            uint64_t a_desc, b_desc;
            if (C::WGRAD) {  // MN-major: 16 K-rows = two 8-row groups = 2048 bytes
              a_desc = smem_desc_sw128(sA + kk * 2048, C::ATOM_BYTES, 1024);
              b_desc = smem_desc_sw128(sB + kk * 2048, C::ATOM_BYTES, 1024);
            } else {         // K-major: 16 bf16 = 32 bytes inside the swizzled row
              a_desc = smem_desc_sw128(sA + kk * 32, 16, 1024);
              b_desc = smem_desc_sw128(sB + kk * 32, 16, 1024);
            }
            tc_mma_f16_pair(d_tmem, a_desc, b_desc, C::IDESC, (kb | kk) != 0 ? 1u : 0u);
          }
          tc_commit_pair_mc(smem_u32(&bars[C::BAR_EMPTY + stage]), 0x3);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit_pair_mc(smem_u32(&bars[C::BAR_TFULL + acc]), 0x3);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      tc_commit_pair(smem_u32(&bars[C::BAR_DRAIN]));
      wait_drain(smem_u32(&bars[C::BAR_DRAIN]), 0, p.timeout_ns);
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ tile scheduler
    if (lane == 0 && leader) tring.schedule<true>(p.tile_counter, num_tiles, wc);
  } else if (warp >= kEpiWarp0) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                    // TMEM lane quarter of this warp
    const int half = (warp - kEpiWarp0) >> 2;  // which 128 of the tile's 256 columns
    const uint32_t tempty_tgt0 = mapa_shared(smem_u32(&bars[C::BAR_TEMPTY]), 0);
    const uint32_t stg = smem_u32(staging) + (warp - kEpiWarp0) * 4096;  // TMA_STORE only
    const uint64_t pol_out = l2_policy_evict_first();
    int acc = 0;
    uint32_t acc_phase = 0;
    int tpos = 0;
    uint32_t tph = 0;
    // One warp's 32x32 fp32 block: row `lane` to the staging slot with 16-byte
    // chunk j at j ^ (lane & 7) (the 128-byte swizzle of the tensor map), then
    // one TMA store. The slot is reused once the previous store has read it.
    auto store_block = [&](const uint32_t (&v)[32], const CUtensorMap* map, int x, int y) {
      if (lane == 0) bulk_wait_read_all();
      __syncwarp();
#pragma unroll
      for (int j = 0; j < 8; ++j)
        st_shared_v4(stg + lane * 128 + ((j ^ (lane & 7)) << 4), v[4 * j], v[4 * j + 1],
                     v[4 * j + 2], v[4 * j + 3]);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_store_2d_hint(map, stg, x, y, pol_out);
        bulk_commit_group();
      }
    };
    for (;;) {
      int tile = 0;
      if (lane == 0) tile = next_tile(tpos, tph);
      tile = __shfl_sync(0xFFFFFFFFu, tile, 0);
      if (tile < 0) break;
      int row0, m, n, l, kblocks;
      if (!tile_info(tile, row0, m, n, l, kblocks)) continue;
      const int lrow0 = static_cast<int>(rank) * 128 + q * 32;  // first TMEM lane of this warp
      auto wg_ptr = [&](int col) -> float* {
        const int64_t orow = static_cast<int64_t>(l) * p.M + m * C::BM + lrow0 + lane;
        return col < p.nsplit ? p.out0 + orow * p.nsplit + col
                              : p.out1 + orow * (p.N - p.nsplit) + (col - p.nsplit);
      };
      if (C::WGRAD && kblocks == 0) {
        // an expert without routes: its gradient is zero (no accumulator used)
        uint32_t z[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) z[i] = 0u;
        for (int c = 0; c < 4; ++c) {
          float* d = wg_ptr(n * C::BN + half * 128 + c * 32);
#pragma unroll
          for (int v = 0; v < 4; ++v) st_global_v8(d + v * 8, z);
        }
        continue;
      }
      if (!wait_bounded(smem_u32(&bars[C::BAR_TFULL + acc]), acc_phase, wc)) break;
      tc_fence_after();
      const uint32_t tbase =
          tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * C::BN);
      uint32_t rv[2][32];
      tmem_ld_32cols(tbase + half * 128, rv[0]);
      tmem_ld_wait();
      if (OP == OP_DGRAD_H) {
        const int64_t row = row0 + lrow0 + lane;
        const int I = p.N;
        const int col0 = n * C::BN + half * 128;
        const float g = __ldg(p.gate_row + row);
        const uint4* ap = reinterpret_cast<const uint4*>(p.ab + row * (2 * I) + col0);
        const uint4* bp = reinterpret_cast<const uint4*>(p.ab + row * (2 * I) + I + col0);
        const uint4* hp = reinterpret_cast<const uint4*>(p.h + row * I + col0);
        uint16_t* dap = p.dab + row * (2 * I) + col0;
        uint16_t* dbp = dap + I;
        uint16_t* hgp = p.hg + row * I + col0;
        float dg = 0.0f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          if (c + 1 < 4) tmem_ld_32cols(tbase + half * 128 + (c + 1) * 32, rv[(c + 1) & 1]);
#pragma unroll
          for (int v = 0; v < 4; ++v) {  // 8 columns per 16-byte vector
            const uint4 av = __ldg(ap + c * 4 + v), bv = __ldg(bp + c * 4 + v),
                        hv = __ldg(hp + c * 4 + v);
            const uint32_t aw[4] = {av.x, av.y, av.z, av.w};
            const uint32_t bw[4] = {bv.x, bv.y, bv.z, bv.w};
            const uint32_t hw[4] = {hv.x, hv.y, hv.z, hv.w};
            uint32_t oa[4], ob[4], oh[4];
#pragma unroll
            for (int w = 0; w < 4; ++w) {
              float da2[2], db2[2], hg2[2];
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                const float dhu = __uint_as_float(rv[c & 1][v * 8 + w * 2 + e]);
                const float a = e ? bf16_hi(aw[w]) : bf16_lo(aw[w]);
                const float b = e ? bf16_hi(bw[w]) : bf16_lo(bw[w]);
                const float hh = e ? bf16_hi(hw[w]) : bf16_lo(hw[w]);
                dg = __fmaf_rn(hh, dhu, dg);
                const float dh = g * dhu;
                const float s = 1.0f / (1.0f + expf(-a));
                da2[e] = dh * b * s * (1.0f + a * (1.0f - s));
                db2[e] = dh * a * s;
                hg2[e] = g * hh;
              }
              oa[w] = pack_bf16x2(da2[0], da2[1]);
              ob[w] = pack_bf16x2(db2[0], db2[1]);
              oh[w] = pack_bf16x2(hg2[0], hg2[1]);
            }
            const int off = c * 32 + v * 8;
            st_global_v4(dap + off, oa[0], oa[1], oa[2], oa[3]);
            st_global_v4(dbp + off, ob[0], ob[1], ob[2], ob[3]);
            st_global_v4(hgp + off, oh[0], oh[1], oh[2], oh[3]);
          }
          if (c + 1 < 4) tmem_ld_wait();
        }
        p.part[row * (I / 128) + n * 2 + half] = dg;
      } else {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          if (c + 1 < 4) tmem_ld_32cols(tbase + half * 128 + (c + 1) * 32, rv[(c + 1) & 1]);
          const int col = n * C::BN + half * 128 + c * 32;
          if (C::WGRAD) {
            float* d = wg_ptr(col);
#pragma unroll
            for (int v = 0; v < 4; ++v)
              st_global_v8(d + v * 8, *reinterpret_cast<const uint32_t(*)[8]>(&rv[c & 1][8 * v]));
          } else {
            store_block(rv[c & 1], &tmY0, col, row0 + lrow0);
          }
          if (c + 1 < 4) tmem_ld_wait();
        }
      }
      // the accumulator may be refilled once every lane's tcgen05.ld completed
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_relaxed_cluster(tempty_tgt0 + acc * 8);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
    if (C::TMA_STORE && lane == 0) bulk_wait_all();  // stores complete before the CTA exits
  }

  __syncthreads();
  cluster_sync();  // the peer no longer reads this CTA's smem or TMEM
  if (tid == 0) finish_tile_counter(p.tile_counter);
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

template <int OP>
cudaError_t launch_bwd(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                       const CUtensorMap& y0, const CUtensorMap& y1, BwdParams p, cudaStream_t s) {
  const size_t smem = bwd_smem_bytes<OP>(p.E);
  if (!p.tile_counter) {  // no counter of the caller's: one from the device's pool
    const cudaError_t e = tile_counter_for_current_device(&p.tile_counter);
    if (e != cudaSuccess) return e;
  }
  return launch_persistent(ffn_bwd_kernel<OP>, 2, smem, s, a, b0, b1, y0, y1, p);
}

BwdParams base_params(const int32_t* offsets, const int32_t* counts, const moe_shape_t& sh,
                      int64_t rows_max, int32_t* dev_status, int* counter) {
  BwdParams p{};
  p.offsets = offsets;
  p.counts = counts;
  p.E = sh.E;
  p.P = sh.P;
  p.rows_max = rows_max;
  p.dev_status = dev_status;
  p.timeout_ns = kWaitTimeoutNs;
  p.tile_counter = counter;
  return p;
}

}  // namespace

cudaError_t launch_expert_ffn_dgrad(const uint16_t* dys, const float* gate_row, const uint16_t* ab,
                                    const uint16_t* h, const uint16_t* W1, const uint16_t* W3,
                                    const uint16_t* W2, const int32_t* offsets,
                                    const int32_t* counts, uint16_t* dab, uint16_t* hg,
                                    float* part, float* dxg, const moe_shape_t& sh,
                                    int64_t rows_max, int32_t* dev_status, cudaStream_t s,
                                    cudaEvent_t ev_mid, int* counter) {
  const int E = sh.E, H = sh.H, I = sh.I;
  const uint64_t EH = static_cast<uint64_t>(E) * H, EI = static_cast<uint64_t>(E) * I;
  CUtensorMap mDys, mW2, mDab, mW1, mW3, mDxg;
  // K-major B operands: the weights as stored, 128 rows x 64 K per box
  if (!make_map(&mDys, dys, H, rows_max, 64, 128) || !make_map(&mW2, W2, H, EI, 64, 128) ||
      !make_map(&mDab, dab, 2ull * I, rows_max, 64, 128) || !make_map(&mW1, W1, I, EH, 64, 128) ||
      !make_map(&mW3, W3, I, EH, 64, 128) || !make_map(&mDxg, dxg, H, rows_max, 32, 32, true))
    return cudaErrorInvalidValue;
  BwdParams p1 = base_params(offsets, counts, sh, rows_max, dev_status, counter);
  p1.K = H;
  p1.N = I;
  p1.ab = ab;
  p1.h = h;
  p1.gate_row = gate_row;
  p1.dab = dab;
  p1.hg = hg;
  p1.part = part;
  cudaError_t e = launch_bwd<OP_DGRAD_H>(mDys, mW2, mW2, mDxg, mDxg, p1, s);
  if (e != cudaSuccess) return e;
  if (ev_mid && (e = cudaEventRecord(ev_mid, s)) != cudaSuccess) return e;
  BwdParams p2 = base_params(offsets, counts, sh, rows_max, dev_status, counter);
  p2.K = 2 * I;
  p2.kswitch = I;
  p2.N = H;
  return launch_bwd<OP_DGRAD_X>(mDab, mW1, mW3, mDxg, mDxg, p2, s);
}

cudaError_t launch_expert_ffn_wgrad(const uint16_t* xg, const uint16_t* dys, const uint16_t* dab,
                                    const uint16_t* hg, const int32_t* offsets,
                                    const int32_t* counts, float* dW1, float* dW3, float* dW2,
                                    const moe_shape_t& sh, int64_t rows_max, int32_t* dev_status,
                                    cudaStream_t s, cudaEvent_t ev_mid, int* counter) {
  const int H = sh.H, I = sh.I;
  CUtensorMap mHg, mDys, mXg, mDab;
  // MN-major operands: 64 columns x 64 rows per box
  if (!make_map(&mHg, hg, I, rows_max, 64, 64) || !make_map(&mDys, dys, H, rows_max, 64, 64) ||
      !make_map(&mXg, xg, H, rows_max, 64, 64) || !make_map(&mDab, dab, 2ull * I, rows_max, 64, 64))
    return cudaErrorInvalidValue;
  BwdParams p1 = base_params(offsets, counts, sh, rows_max, dev_status, counter);
  p1.M = I;
  p1.N = H;
  p1.nsplit = H;
  p1.out0 = p1.out1 = dW2;
  // the output maps are unused: the weight gradients are stored directly
  cudaError_t e = launch_bwd<OP_WGRAD>(mHg, mDys, mDys, mHg, mHg, p1, s);
  if (e != cudaSuccess) return e;
  if (ev_mid && (e = cudaEventRecord(ev_mid, s)) != cudaSuccess) return e;
  BwdParams p2 = base_params(offsets, counts, sh, rows_max, dev_status, counter);
  p2.M = H;
  p2.N = 2 * I;
  p2.nsplit = I;
  p2.out0 = dW1;
  p2.out1 = dW3;
  return launch_bwd<OP_WGRAD>(mXg, mDab, mDab, mXg, mXg, p2, s);
}

}  // namespace moe
