// MXFP8 routed experts: the grouped SwiGLU expert FFN on E4M3 operands with
// E8M0 block scales, on the block-scaled 5th-generation tensor cores.
//
// "Mixture-of-Kittens: A MoE Megakernel for GB300 NVL72", section 5 (MXFP8
// routed experts; the quantisation fused into the dispatch and into the
// SwiGLU epilogue); the OCP Microscaling formats (E4M3 elements, one E8M0
// scale per 32 values along the reduction dimension). For each expert l and
// its rows [S[l], S[l+1]) of the gathered, quantised tokens:
//   GEMM1  acc = mx(x) . [mx(W1[l]) | mx(W3[l])]          fp32 in TMEM
//          h = silu(acc_W1) * acc_W3 (fp32), quantised to MXFP8 along I
//          (one scale per 32 h columns) by the epilogue
//   GEMM2  y = mx(h) . mx(W2[l])                           fp32
// where mx(v) is the value the codes stand for: code value x 2^(scale - 127).
//
// Operands, all K-major (the reduction dimension contiguous):
//   A   xq [rows, H] (GEMM1), hq [rows, I] (GEMM2): E4M3 codes
//   B   the weights transposed once: W1t, W3t [E, I, H]; W2t [E, H, I]
//   scales of every operand in the tiled layout of mx_tiled_offset
//   (internal.cuh): 512-byte atoms of 128 rows x 4 blocks of 32 values.
//
// Design: the forward FFN's persistent warp-specialised CTA-pair kernel
// (expert_ffn.cu) with the block-scaled MMA
// (tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale, M = 256, K = 32 per
// instruction). A pipeline stage holds 128 K values (one 128-byte swizzled
// row per operand row, four MMAs) and their scales: one 512-byte atom for the
// CTA's 128 A rows and one atom per 128 columns of the tile (each CTA of the
// pair needs the scales of every column its rows meet). The producer loads
// codes and scale atoms with TMA (pair form; each CTA fetches its own copy).
// The MMA thread moves a stage's scales into TMEM with tcgen05.cp (32x128b,
// replicated into the four lane quarters: 4 columns per atom) and then issues
// the stage's four MMAs, each naming its scale byte (0..3) of the 32-bit
// cells. Scale slots in TMEM follow the smem stages: a slot is rewritten only
// after the MMAs that read it completed (the stage's empty barrier came
// first). TMEM holds the accumulators and STAGES x 8 or 16 scale columns:
//   GEMM1  256 x 256 tiles (128 h columns through W1 and W3, CTA 0 holding
//          W1's rows and CTA 1 W3's), one 256-column accumulator: a second
//          would leave no columns for the scales; each epilogue thread reads
//          both of its MX blocks (128 values) into registers and releases the
//          accumulator before their arithmetic, so the next tile's MMAs wait
//          only for the TMEM reads (it writes 1 byte per h value, against a
//          56-stage K loop);
//   GEMM2  256 x 256 tiles (CTA r holding W2's columns 128 r .. +128), one
//          256-column accumulator: each epilogue thread reads its 128
//          accumulator values into registers and releases the accumulator
//          before it stages and stores them, so the next tile's MMAs wait
//          only for the TMEM reads. A block-scaled MMA of N = 128 takes as long
//          to issue as one of N = 256, so the wider tile halves GEMM2's MMAs.
//
// Every output element is produced by one CTA pair in a fixed K order (no
// split-K, no atomics): the result is deterministic and independent of which
// other rows share the launch. Every mbarrier wait is bounded; on a timeout
// all roles unwind, in-flight copies and MMAs are drained with a bounded
// wait, TMEM is freed and MOE_DEV_TIMEOUT is raised.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "internal.cuh"
#include "mx_block.cuh"
#include "persistent_gemm.cuh"
#include "sm100.cuh"
#include "sm100_mx.cuh"

namespace moe {
namespace {

using namespace sm100;
using namespace pg;

// MODE 0: GEMM1 + SwiGLU + MX quantisation of h. MODE 1: GEMM2 -> fp32 y.
template <int MODE>
struct MxCfg {
  static constexpr bool TMA_STORE = MODE == 1;
  static constexpr int STAGING_BYTES = TMA_STORE ? 8 * 2048 : 0;  // 8 warps x 32x16 fp32
  static constexpr int BM = 256;
  static constexpr int BN = 256;                       // accumulator columns per tile
  static constexpr int ACC = 1;                        // accumulators in TMEM
  static constexpr int BK = 128;                       // E4M3 values (bytes) per stage
  static constexpr int MMA_K = 32;                     // K of one block-scaled MMA
  static constexpr int B_ROWS = BN / 2;                // B rows (tile columns) per CTA
  static constexpr int A_BYTES = 128 * BK;             // this CTA's 128 rows
  static constexpr int B_BYTES = B_ROWS * BK;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;  // 32 KB
  static constexpr int SFB_ATOMS = BN / 128;             // scale atoms of the tile's columns
  static constexpr int SF_STAGE_BYTES = 512 * (1 + SFB_ATOMS);
  static constexpr int STAGES = 6;
  static constexpr int TMEM_SF = ACC * BN;              // scale columns follow the accumulators
  static constexpr int SF_COLS = 4 * (1 + SFB_ATOMS) <= 8 ? 8 : 16;  // A at +0, B at +4
  static_assert(TMEM_SF + STAGES * SF_COLS <= kTmemCols, "TMEM budget");
  static constexpr uint32_t IDESC = idesc_mxf8_e4m3(BM, BN, 0, 0);
  static constexpr int BAR_FULL = 0;
  static constexpr int BAR_EMPTY = STAGES;
  static constexpr int BAR_TFULL = 2 * STAGES;
  static constexpr int BAR_TEMPTY = 2 * STAGES + ACC;
  static constexpr int BAR_DRAIN = 2 * STAGES + 2 * ACC;
  static constexpr int BAR_TID_FULL = BAR_DRAIN + 1;
  static constexpr int BAR_TID_EMPTY = BAR_TID_FULL + kRing;
  static constexpr int NUM_BARS = BAR_TID_EMPTY + kRing;
  // readers of each tile id: producer, MMA issuer and 8 epilogue warps of the
  // leader; producer and 8 epilogue warps of the follower
  static constexpr int TID_CONSUMERS = 19;
  static_assert(STAGE_BYTES % 1024 == 0 && A_BYTES % 1024 == 0, "swizzle atoms stay 1024-aligned");
  static_assert(BK / MMA_K == 4, "one 32-bit TMEM scale cell per row and stage");
};

struct MxParams {
  int* tile_counter;       // {next tile to hand out, CTAs finished}; zero at launch
  const int32_t* offsets;  // [E+1] segment starts (multiples of 256)
  const int32_t* counts;   // [E, P] or null
  int32_t E, P;
  int32_t K;               // reduction length: H (GEMM1), I (GEMM2)
  int32_t Nout;            // output row length: I (GEMM1), H (GEMM2)
  int64_t rows_max;
  uint8_t* hq;             // GEMM1: h codes [rows_max, I]
  uint8_t* hs;             // GEMM1: h scales, tiled over [rows_max, I/32]
  int32_t* dev_status;
  int64_t timeout_ns;
  // LAND (GEMM1): the quantising pull dispatch inside the kernel
  const int2* phi;         // [rows_max] (src_rank, src_idx)
  int32_t n_per_peer;      // N (token row = src_rank * N + src_idx)
  const void* x;           // token activations bf16 [P*N, H]
  uint8_t* xq;             // the A operand's codes [rows_max, H] the tensor map reads
  uint8_t* xs;             // its scales, tiled over [rows_max, H/32]
  int* land_next;          // next 128-row block to land (0 at launch)
  int* land_ready;         // [rows_max / 128] block-landed flags (0 at launch)
};

template <int MODE>
size_t mx_smem_bytes(int E) {
  using C = MxCfg<MODE>;
  return 1024 + static_cast<size_t>(C::STAGES) * (C::STAGE_BYTES + C::SF_STAGE_BYTES) +
         C::STAGING_BYTES + C::NUM_BARS * 8 + 16 + kRing * 4 + static_cast<size_t>(2 * E + 1) * 4;
}

__device__ __forceinline__ float silu(float a) { return a / (1.0f + expf(-a)); }

// floor(log2 v) of a finite positive fp32, exactly (subnormals included).
__device__ __forceinline__ int f32_floor_log2(float v) {
  const uint32_t bits = __float_as_uint(v);
  const int ef = static_cast<int>(bits >> 23);
  if (ef != 0) return ef - 127;
  return -149 + (31 - __clz(bits & 0x7FFFFFu));  // subnormal: mantissa x 2^-149
}

// MX quantisation of 32 fp32 values (one block): E4M3 codes in element order
// (four per word, the lowest element in the low byte) and the E8M0 scale code.
// The same rule as the dispatch's quantisation, applied to fp32 inputs.
__device__ __forceinline__ void mx_block_f32(const float (&v)[32], uint32_t (&codes)[8],
                                             uint8_t& scale) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
  int e = -127;
  if (amax > 0.0f) e = max(-127, min(127, f32_floor_log2(amax) - 8));
  scale = static_cast<uint8_t>(e + 127);
  const float inv = __int_as_float((127 - e) << 23);  // 2^-e, a normal fp32 for e in [-127, 119]
#pragma unroll
  for (int w = 0; w < 8; ++w) {
    const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(
        make_float2(v[4 * w] * inv, v[4 * w + 1] * inv), __NV_SATFINITE, __NV_E4M3);
    const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(
        make_float2(v[4 * w + 2] * inv, v[4 * w + 3] * inv), __NV_SATFINITE, __NV_E4M3);
    codes[w] = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
  }
}

// LAND (MODE 0): the quantising pull dispatch runs inside this kernel, as in
// the bf16 FFN: warp 3 of every CTA takes 128-row blocks of the
// expert-sorted layout in order from a device counter, quantises each row
// x[Phi[row]] by the MX block rule (mx_block.cuh) into the codes and tiled
// scales the A tensor maps read (padding rows: zero codes, scale code 0), and
// publishes the block with a release store of its flag. The TMA producer
// waits (bounded) for the flag of its CTA's 128 rows before it loads a tile's
// A codes and scales, then issues a cross-proxy fence (the rows were written
// through the generic proxy, TMA reads through the async proxy).
template <int MODE, bool LAND = false>
__global__ void __launch_bounds__(kNumThreads, 1)
    ffn_mx_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmSA,
                  const __grid_constant__ CUtensorMap tmB0, const __grid_constant__ CUtensorMap tmSB0,
                  const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ CUtensorMap tmSB1,
                  const __grid_constant__ CUtensorMap tmY, const MxParams p) {
  using C = MxCfg<MODE>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* staging = smem + C::STAGES * C::STAGE_BYTES;  // TMA_STORE only (1024-aligned)
  uint8_t* sf = staging + C::STAGING_BYTES;              // [STAGES] x {A atom, B atoms}
  uint64_t* bars = reinterpret_cast<uint64_t*>(sf + C::STAGES * C::SF_STAGE_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NUM_BARS);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  int* bad_flag = abort_flag + 1;
  int* tile_ring = reinterpret_cast<int*>(tmem_slot + 4);
  int32_t* s_off = reinterpret_cast<int32_t*>(tile_ring + kRing);  // [E+1]
  int32_t* s_end = s_off + (p.E + 1);                            // [E]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int E = p.E;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;

  if (tid == 0) {
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(smem_u32(&bars[C::BAR_FULL + i]), 1);
      mbar_init(smem_u32(&bars[C::BAR_EMPTY + i]), 1);
    }
    for (int i = 0; i < C::ACC; ++i) {
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
    tma_prefetch_desc(&tmSA);
    tma_prefetch_desc(&tmB0);
    tma_prefetch_desc(&tmSB0);
    tma_prefetch_desc(&tmB1);
    tma_prefetch_desc(&tmSB1);
    if (C::TMA_STORE) tma_prefetch_desc(&tmY);
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

  const int rows_used = bad_sched ? 0 : s_off[E];
  // GEMM1: a tile's 256 accumulator columns are 128 h columns seen through W1
  // and W3; GEMM2: 256 y columns
  const int tiles_n = p.Nout / (MODE == 0 ? 128 : C::BN);
  const int num_tiles = (rows_used / C::BM) * tiles_n;
  const int kblocks = p.K / C::BK;  // stages per tile = scale atoms per 128-row block
  const WaitCtx wc{abort_flag, p.dev_status, p.timeout_ns, MOE_DEV_TIMEOUT};

  const uint32_t tid_empty_local = smem_u32(&bars[C::BAR_TID_EMPTY]);
  const TileRing tring{tile_ring, smem_u32(&bars[C::BAR_TID_FULL]), tid_empty_local,
                       mapa_shared(tid_empty_local, 0), !leader};
  auto next_tile = [&](int& pos, uint32_t& ph) -> int { return tring.next<true>(pos, ph, wc); };
  const int64_t drain_ns = p.timeout_ns < 100000000ll ? p.timeout_ns : 100000000ll;
  // tile -> (first row, n-tile, expert); the forward FFN's grouped raster
  auto tile_info = [&](int tile, int& row0, int& n, int& l) -> bool {
    return grouped_row_tile<C::BM, 8, 1>(tile, s_off, s_end, E, tiles_n, row0, n, l);
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
        int row0, n, l;
        if (!tile_info(tile, row0, n, l)) continue;
        const int arow = row0 + static_cast<int>(rank) * 128;
        // B rows (of the transposed weights) this tile meets: GEMM1: W1t and
        // W3t rows l*I + n*128 .. +128 (CTA 0 loads W1t's, CTA 1 W3t's);
        // GEMM2: W2t rows l*H + n*256 .. +256 (CTA r loads 128 r .. +128).
        // Either way one scale atom per 128 rows, two per tile.
        const int brow = l * p.Nout + n * (MODE == 0 ? 128 : C::BN);
        if (LAND) {  // this CTA's 128 A rows must have landed
          if (!wait_flag_bounded(p.land_ready + arow / 128, wc)) break;
          asm volatile("fence.proxy.async.global;" ::: "memory");
        }
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!wait_bounded(smem_u32(&bars[C::BAR_EMPTY + stage]), phase ^ 1u, wc)) {
            ok = false;
            break;
          }
          const uint32_t full_tgt = full_tgt0 + stage * 8;
          const uint32_t sA = smem_u32(smem + stage * C::STAGE_BYTES);
          const uint32_t sB = sA + C::A_BYTES;
          const uint32_t sSA = smem_u32(sf + stage * C::SF_STAGE_BYTES);
          const uint32_t sSB = sSA + 512;
          const int kx = kb * C::BK;
          if (leader) mbar_arrive_expect_tx(full0 + stage * 8, 2 * (C::STAGE_BYTES + C::SF_STAGE_BYTES));
          tma_load_2d_pair(sA, &tmA, kx, arow, full_tgt);
          tma_load_2d_pair(sSA, &tmSA, 0, (arow / 128) * kblocks + kb, full_tgt);
          if (MODE == 0) {
            tma_load_2d_pair(sB, rank == 1 ? &tmB1 : &tmB0, kx, brow, full_tgt);
            tma_load_2d_pair(sSB, &tmSB0, 0, (brow / 128) * kblocks + kb, full_tgt);
            tma_load_2d_pair(sSB + 512, &tmSB1, 0, (brow / 128) * kblocks + kb, full_tgt);
          } else {
            tma_load_2d_pair(sB, &tmB0, kx, brow + static_cast<int>(rank) * C::B_ROWS, full_tgt);
            tma_load_2d_pair(sSB, &tmSB0, 0, (brow / 128) * kblocks + kb, full_tgt);
            tma_load_2d_pair(sSB + 512, &tmSB0, 0, (brow / 128 + 1) * kblocks + kb, full_tgt);
          }
          ++issued;
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // no load may still be landing in shared memory when the CTA exits
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
        int row0, n, l;
        if (!tile_info(tile, row0, n, l)) continue;
        // an accumulator is free once both CTAs' epilogues drained it
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
          const uint32_t sSA = smem_u32(sf + stage * C::SF_STAGE_BYTES);
          const uint32_t sSB = sSA + 512;
          const uint32_t tsf = tmem_base + static_cast<uint32_t>(C::TMEM_SF + stage * C::SF_COLS);
          // 32 rows x 16 bytes per copy: four 8-row core matrices 128 bytes
          // apart. A's atom -> columns +0..3; B's atoms -> +4..7 (+8..11):
          // tile column c reads its scales at column +4 + c/32
          tc_cp_pair_32x128b_x4(tsf, smem_desc_noswz(sSA, 128));
#pragma unroll
          for (int a = 0; a < C::SFB_ATOMS; ++a)
            tc_cp_pair_32x128b_x4(tsf + 4 + 4 * a, smem_desc_noswz(sSB + 512 * a, 128));
#pragma unroll
          for (int kk = 0; kk < C::BK / C::MMA_K; ++kk) {
            // K-major: 32 E4M3 = 32 bytes inside the 128-byte swizzled row
            const uint64_t a_desc = smem_desc_sw128(sA + kk * 32, 16, 1024);
            const uint64_t b_desc = smem_desc_sw128(sB + kk * 32, 16, 1024);
            const uint32_t sel = static_cast<uint32_t>(kk);
            const uint32_t idesc = C::IDESC | (sel << 29) | (sel << 4);
            tc_mma_mx_pair(d_tmem, a_desc, b_desc, idesc, tsf | (sel << 30),
                           (tsf + 4) | (sel << 30), (kb | kk) != 0 ? 1u : 0u);
          }
          tc_commit_pair_mc(smem_u32(&bars[C::BAR_EMPTY + stage]), 0x3);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit_pair_mc(smem_u32(&bars[C::BAR_TFULL + acc]), 0x3);
        if (++acc == C::ACC) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      tc_commit_pair(smem_u32(&bars[C::BAR_DRAIN]));
      wait_drain(smem_u32(&bars[C::BAR_DRAIN]), 0, p.timeout_ns);
    }
  } else if (warp == 3 && LAND) {
    // ------------------------------------------------------------ quantising pull dispatch
    const int nblk = rows_used / 128;
    const int kb32 = p.K / 32;  // MX blocks of a row
    const uint4* xsrc = reinterpret_cast<const uint4*>(p.x);
    int bad = 0;
    for (;;) {
      int b = 0;
      if (lane == 0) b = atomicAdd(p.land_next, 1);
      b = __shfl_sync(0xFFFFFFFFu, b, 0);
      if (b >= nblk || *wc.abort) break;
      constexpr int U = 7;  // blocks per lane in one round: a 7,168-wide row (224 blocks)
      if (2 * kb32 <= 32 * U) {
        // rows of at most 3,584 values, whole rows per round: lane j takes
        // blocks j, j+32, ... of the round's rows back to back (block f of
        // the round: row f / kb32, block f % kb32), so the rows share a round
        // instead of each costing a memory round trip
        const int rpr = (32 * U) / kb32;  // 2 .. 28
#pragma unroll 1
        for (int rr0 = 0; rr0 < 128; rr0 += rpr) {
          // lane l < rpr looks up row rr0 + l once: the 16-byte offset of its
          // token row, -1 for padding; each block takes its row's by shuffle
          int64_t so_l = -1;
          if (lane < rpr && rr0 + lane < 128) {
            const int2 e = __ldg(p.phi + static_cast<int64_t>(b) * 128 + rr0 + lane);
            const bool v = e.x >= 0 && e.x < p.P && e.y >= 0 && e.y < p.n_per_peer;
            if (!v && (e.x >= 0 || e.y != -1)) bad = 1;  // (-1,-1) is padding
            if (v) so_l = (static_cast<int64_t>(e.x) * p.n_per_peer + e.y) * (p.K / 8);
          }
          uint4 in[U][4];
#pragma unroll
          for (int u = 0; u < U; ++u) {
            const int f = lane + 32 * u;
            const int ro = min(f / kb32, 31), blk = f - (f / kb32) * kb32;
            const int64_t so = __shfl_sync(0xFFFFFFFFu, so_l, ro);
            const bool ld = f < rpr * kb32 && so >= 0;
#pragma unroll
            for (int c = 0; c < 4; ++c)
              in[u][c] = ld ? __ldg(xsrc + so + blk * 4 + c) : make_uint4(0, 0, 0, 0);
          }
#pragma unroll
          for (int u = 0; u < U; ++u) {
            const int f = lane + 32 * u;
            const int ro = f / kb32, blk = f - ro * kb32;
            if (f < rpr * kb32 && rr0 + ro < 128) {
              const int64_t row = static_cast<int64_t>(b) * 128 + rr0 + ro;
              uint4 out[2];
              uint8_t scale;
              mx::mx_block(in[u], out, scale);
              uint4* qrow = reinterpret_cast<uint4*>(p.xq) + row * (p.K / 16);
              qrow[blk * 2] = out[0];
              qrow[blk * 2 + 1] = out[1];
              p.xs[mx_tiled_offset(row, blk, kb32)] = scale;
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
          const uint4* src =
              xsrc + (v ? (static_cast<int64_t>(e.x) * p.n_per_peer + e.y) * (p.K / 8) : 0);
          uint4* qrow = reinterpret_cast<uint4*>(p.xq) + row * (p.K / 16);
          // lane j takes blocks j, j+32, ...: a 7,168-wide row in one round of
          // 28 16-byte loads per lane
#pragma unroll 1
          for (int b0 = lane; b0 < kb32; b0 += 32 * U) {
            uint4 in[U][4];
#pragma unroll
            for (int u = 0; u < U; ++u) {
              const int blk = b0 + 32 * u;
#pragma unroll
              for (int c = 0; c < 4; ++c)
                in[u][c] = (v && blk < kb32) ? __ldg(src + blk * 4 + c) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
              const int blk = b0 + 32 * u;
              if (blk < kb32) {
                uint4 out[2];
                uint8_t scale;
                mx::mx_block(in[u], out, scale);
                qrow[blk * 2] = out[0];
                qrow[blk * 2 + 1] = out[1];
                p.xs[mx_tiled_offset(row, blk, kb32)] = scale;
              }
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
  } else if (warp == 2) {
    // ------------------------------------------------------------ tile scheduler
    if (lane == 0 && leader) tring.schedule<true>(p.tile_counter, num_tiles, wc);
  } else if (warp >= kEpiWarp0) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                    // TMEM lane quarter of this warp
    const int half = (warp - kEpiWarp0) >> 2;  // which half of the tile's columns
    const uint32_t tempty_tgt0 = mapa_shared(smem_u32(&bars[C::BAR_TEMPTY]), 0);
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
      if (MODE == 0) {
        // accumulator columns [0,128) = x.W1, [128,256) = x.W3 for h columns
        // n*128 + j; this warp's 64 columns are two 32-column MX blocks of h.
        // Both blocks are read into registers first and the single
        // accumulator is released, so the next tile's MMAs overlap the
        // SwiGLU, quantisation and stores of both.
        const int I = p.Nout;
        uint32_t ra[2][32], rb[2][32];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          tmem_ld_32cols(tbase + half * 64 + c * 32, ra[c]);
          tmem_ld_32cols(tbase + 128 + half * 64 + c * 32, rb[c]);
        }
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_relaxed_cluster(tempty_tgt0 + acc * 8);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          float hv[32];
#pragma unroll
          for (int i = 0; i < 32; ++i)
            hv[i] = silu(__uint_as_float(ra[c][i])) * __uint_as_float(rb[c][i]);
          uint32_t codes[8];
          uint8_t scale;
          mx_block_f32(hv, codes, scale);
          const int col = n * 128 + half * 64 + c * 32;
          st_global_v8(p.hq + row * I + col, codes);
          p.hs[mx_tiled_offset(row, col / 32, I / 32)] = scale;
        }
      } else {
        // this warp's 128 of the tile's 256 columns, read whole into
        // registers; the accumulator is released before the stores. Row
        // `lane` of each 32x16 block then goes to the warp's 2 KB staging slot
        // with 16-byte chunk j at j ^ ((lane >> 1) & 3) (the tensor map's
        // 64-byte swizzle) and leaves with one TMA store; the slot is reused
        // once the previous store has read it.
        uint32_t rv[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld_32cols(tbase + half * 128 + c * 32, rv[c]);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_relaxed_cluster(tempty_tgt0 + acc * 8);
        const uint32_t stg = smem_u32(staging) + (warp - kEpiWarp0) * 2048;
        const uint64_t pol_y = l2_policy_evict_first();
        const int ycol = n * C::BN + half * 128;
        const int yrow0 = row0 + static_cast<int>(rank) * 128 + q * 32;
        // a 32-row block wholly past the expert's routes holds only padding
        // rows, which nothing reads: its y is not written
        const int nblk = yrow0 < s_end[l] ? 8 : 0;
#pragma unroll
        for (int c = 0; c < nblk; ++c) {
          if (lane == 0) bulk_wait_read_all();
          __syncwarp();
#pragma unroll
          for (int j = 0; j < 4; ++j)
            st_shared_v4(stg + lane * 64 + ((j ^ ((lane >> 1) & 3)) << 4),
                         rv[c >> 1][(c & 1) * 16 + 4 * j], rv[c >> 1][(c & 1) * 16 + 4 * j + 1],
                         rv[c >> 1][(c & 1) * 16 + 4 * j + 2], rv[c >> 1][(c & 1) * 16 + 4 * j + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {  // y is streamed out and read once, by the combine
            tma_store_2d_hint(&tmY, stg, ycol + c * 16, yrow0, pol_y);
            bulk_commit_group();
          }
        }
      }
      // (both modes released the accumulator above, once every lane's
      // tcgen05.ld had completed)
      if (++acc == C::ACC) {
        acc = 0;
        acc_phase ^= 1u;
      }
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

template <int MODE, bool LAND = false>
cudaError_t launch_mx(const CUtensorMap& a, const CUtensorMap& sa, const CUtensorMap& b0,
                      const CUtensorMap& sb0, const CUtensorMap& b1, const CUtensorMap& sb1,
                      const CUtensorMap& y, MxParams p, cudaStream_t s) {
  const size_t smem = mx_smem_bytes<MODE>(p.E);
  if (!p.tile_counter) {  // no counter of the caller's: one from the device's pool
    const cudaError_t e = tile_counter_for_current_device(&p.tile_counter);
    if (e != cudaSuccess) return e;
  }
  return launch_persistent(ffn_mx_kernel<MODE, LAND>, 2, smem, s, a, sa, b0, sb0, b1, sb1, y, p);
}

}  // namespace

cudaError_t launch_expert_ffn_mxfp8(const uint8_t* xq, const uint8_t* xs, const uint8_t* W1q,
                                    const uint8_t* W1s, const uint8_t* W3q, const uint8_t* W3s,
                                    const uint8_t* W2q, const uint8_t* W2s,
                                    const int32_t* offsets, const int32_t* counts, uint8_t* hq,
                                    uint8_t* hs, float* y, const moe_shape_t& sh,
                                    int64_t rows_max, int32_t* dev_status, cudaStream_t s,
                                    cudaEvent_t ev_mid, int* counter, const LandArgs* land) {
  const int E = sh.E, H = sh.H, I = sh.I;
  const uint64_t EH = static_cast<uint64_t>(E) * H, EI = static_cast<uint64_t>(E) * I;
  const uint64_t rb = static_cast<uint64_t>(rows_max) / 128;  // 128-row blocks of the activations
  CUtensorMap mXq, mXs, mW1, mW1s, mW3, mW3s, mHq, mHs, mW2, mW2s, mY;
  if (!make_map_u8(&mXq, xq, H, rows_max, 128, 128) || !make_map_sf_atoms(&mXs, xs, rb * (H / 128)) ||
      !make_map_u8(&mW1, W1q, H, EI, 128, 128) ||
      !make_map_sf_atoms(&mW1s, W1s, EI / 128 * (H / 128)) ||
      !make_map_u8(&mW3, W3q, H, EI, 128, 128) ||
      !make_map_sf_atoms(&mW3s, W3s, EI / 128 * (H / 128)) ||
      !make_map_u8(&mHq, hq, I, rows_max, 128, 128) || !make_map_sf_atoms(&mHs, hs, rb * (I / 128)) ||
      !make_map_u8(&mW2, W2q, I, EH, 128, 128) ||  // GEMM2: 128 B rows per CTA
      !make_map_sf_atoms(&mW2s, W2s, EH / 128 * (I / 128)) ||
      !make_map(&mY, y, H, rows_max, 16, 32, true, true))
    return cudaErrorInvalidValue;
  MxParams p1{counter, offsets, counts, E, sh.P, H, I, rows_max, hq, hs, dev_status, kWaitTimeoutNs};
  cudaError_t e;
  if (land) {  // the quantising pull dispatch lands xq, xs inside GEMM1
    p1.phi = reinterpret_cast<const int2*>(land->phi);
    p1.n_per_peer = sh.N;
    p1.x = land->x;
    p1.xq = const_cast<uint8_t*>(xq);
    p1.xs = const_cast<uint8_t*>(xs);
    p1.land_next = land->next;
    p1.land_ready = land->ready;
    e = launch_mx<0, true>(mXq, mXs, mW1, mW1s, mW3, mW3s, mY, p1, s);
  } else {
    e = launch_mx<0>(mXq, mXs, mW1, mW1s, mW3, mW3s, mY, p1, s);
  }
  if (e != cudaSuccess) return e;
  if (ev_mid && (e = cudaEventRecord(ev_mid, s)) != cudaSuccess) return e;
  MxParams p2{counter, offsets, counts, E, sh.P, I, H, rows_max, nullptr, nullptr, dev_status,
              kWaitTimeoutNs};
  return launch_mx<1>(mHq, mHs, mW2, mW2s, mW2, mW2s, mY, p2, s);
}

}  // namespace moe
