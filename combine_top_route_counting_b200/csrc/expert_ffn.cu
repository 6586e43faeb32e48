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
// Design (one persistent CTA per SM, 256 threads, warp-specialised):
//   warp 0      TMA producer: 4-stage ring of {A 128x64, B 64x256} bf16
//               tiles, 128-byte swizzle, mbarrier complete_tx
//   warp 1      TMEM allocator and MMA issuer: tcgen05.mma kind::f16,
//               M=128 N=256 K=16, A K-major, B MN-major (the weights are
//               stored [K, N] with N contiguous, so no transpose is needed)
//   warps 4-7   epilogue: tcgen05.ld of the fp32 accumulator (one TMEM lane
//               per row), SwiGLU or fp32 store to global memory
//   TMEM        2 x 256 fp32 columns: the accumulator of tile i+1 fills while
//               the epilogue drains tile i
// A 128-row M-tile never straddles two experts because every segment is a
// multiple of 128 rows; the expert of a tile comes from a binary search over
// the segment offsets held in shared memory. Tiles holding only padding rows
// are skipped. Tiles are visited m-major, so the CTAs running at one time
// share an expert's weights and the A rows of a few M-tiles through L2.
//
// Every output element is produced by one CTA with a fixed K order (no
// split-K, no atomics): the result is bitwise deterministic and independent
// of which other rows share the launch.
//
// Every mbarrier wait is bounded (sm100.cuh): if any wait gives up, all roles
// unwind, in-flight TMA loads and MMAs are drained with a bounded wait, TMEM
// is freed and MOE_DEV_TIMEOUT is raised.
#include <cuda_bf16.h>

#include <mutex>

#include "internal.cuh"
#include "sm100.cuh"

namespace moe {
namespace {

using namespace sm100;

constexpr int BM = 128;
constexpr int BN = 256;  // accumulator columns per tile
constexpr int BK = 64;   // K per stage: one 128-byte swizzle row of bf16
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;             // 16 KB
constexpr int B_ATOM_BYTES = 64 * BK * 2;        // one 64-column x 64-K box: 8 KB
constexpr int B_BYTES = (BN / 64) * B_ATOM_BYTES;  // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;   // 48 KB
constexpr int NUM_THREADS = 256;
constexpr int TMEM_COLS = 512;                   // 2 accumulators x 256 columns
constexpr int UMMA_K = 16;
constexpr uint32_t IDESC = idesc_bf16_f32(BM, BN, /*B MN-major*/ 1);
static_assert(STAGE_BYTES % 1024 == 0 && A_BYTES % 1024 == 0, "swizzle atoms stay 1024-aligned");

// barrier slots
constexpr int BAR_FULL = 0;
constexpr int BAR_EMPTY = STAGES;
constexpr int BAR_TFULL = 2 * STAGES;
constexpr int BAR_TEMPTY = 2 * STAGES + 2;
constexpr int BAR_DRAIN = 2 * STAGES + 4;
constexpr int NUM_BARS = 2 * STAGES + 5;

struct FfnParams {
  const int32_t* offsets;  // [E+1]
  const int32_t* counts;   // [E, P] or null
  int32_t E, P;
  int32_t K;               // reduction length (H for GEMM1, I for GEMM2)
  int32_t Nout;            // output row length (I for GEMM1, H for GEMM2)
  int64_t rows_max;
  void* out;               // bf16 h [rows_max, I] or fp32 y [rows_max, H]
  int32_t* dev_status;
  int64_t timeout_ns;
};

size_t smem_bytes_for(int E) {
  return 1024 /*alignment slack*/ + static_cast<size_t>(STAGES) * STAGE_BYTES +
         NUM_BARS * 8 + 16 + static_cast<size_t>(2 * E + 1) * 4;
}

__device__ __forceinline__ float silu(float a) { return a / (1.0f + expf(-a)); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat16 a = __float2bfloat16_rn(lo);
  const __nv_bfloat16 b = __float2bfloat16_rn(hi);
  return static_cast<uint32_t>(__bfloat16_as_ushort(a)) |
         (static_cast<uint32_t>(__bfloat16_as_ushort(b)) << 16);
}

// MODE 0: GEMM1 + SwiGLU -> bf16 h. MODE 1: GEMM2 -> fp32 y.
template <int MODE>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    ffn_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                    const __grid_constant__ CUtensorMap tmB1, const FfnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NUM_BARS);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  int* bad_flag = abort_flag + 1;
  int32_t* s_off = reinterpret_cast<int32_t*>(tmem_slot + 4);  // [E+1] segment starts
  int32_t* s_end = s_off + (p.E + 1);                            // [E] end of real rows

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int E = p.E;

  if (tid == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(smem_u32(&bars[BAR_FULL + i]), 1);
      mbar_init(smem_u32(&bars[BAR_EMPTY + i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&bars[BAR_TFULL + i]), 1);
      mbar_init(smem_u32(&bars[BAR_TEMPTY + i]), 128);
    }
    mbar_init(smem_u32(&bars[BAR_DRAIN]), 1);
    *abort_flag = 0;
    *bad_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB0);
    tma_prefetch_desc(&tmB1);
  }
  for (int l = tid; l <= E; l += NUM_THREADS) s_off[l] = __ldg(p.offsets + l);
  __syncthreads();
  for (int l = tid; l < E; l += NUM_THREADS) {
    const int a = s_off[l], b = s_off[l + 1];
    bool bad = a < 0 || b < a || (a & (BM - 1)) || (b & (BM - 1)) || b > p.rows_max;
    int T = b - a;
    if (p.counts) {
      int t = 0;
      for (int r = 0; r < p.P; ++r) t += __ldg(p.counts + l * p.P + r);
      if (t < 0 || t > b - a) bad = true;
      else T = t;
    }
    if (bad) *bad_flag = 1;
    s_end[l] = a + T;
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const bool bad_sched = *bad_flag != 0;
  if (bad_sched && tid == 0) atomicOr(p.dev_status, MOE_DEV_BAD_SCHEDULE);

  const int rows_used = bad_sched ? 0 : s_off[E];
  const int tiles_n = (MODE == 0) ? p.Nout / 128 : p.Nout / BN;
  const int num_tiles = (rows_used / BM) * tiles_n;
  const int kblocks = p.K / BK;
  const WaitCtx wc{abort_flag, p.dev_status, p.timeout_ns, MOE_DEV_TIMEOUT};

  // tile -> (first row, n-tile, expert); false if the tile holds only padding
  auto tile_info = [&](int tile, int& row0, int& n, int& l) -> bool {
    const int m = tile / tiles_n;
    n = tile - m * tiles_n;
    row0 = m * BM;
    int lo = 0, hi = E - 1;  // largest l with s_off[l] <= row0
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_off[mid] <= row0) lo = mid;
      else hi = mid - 1;
    }
    l = lo;
    return row0 < s_end[l];
  };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int64_t issued = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
        int row0, n, l;
        if (!tile_info(tile, row0, n, l)) continue;
        const int yb = l * p.K;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!wait_bounded(smem_u32(&bars[BAR_EMPTY + stage]), phase ^ 1u, wc)) {
            ok = false;
            break;
          }
          const uint32_t full = smem_u32(&bars[BAR_FULL + stage]);
          const uint32_t sA = smem_u32(smem + stage * STAGE_BYTES);
          const uint32_t sB = sA + A_BYTES;
          mbar_arrive_expect_tx(full, STAGE_BYTES);
          tma_load_2d(sA, &tmA, kb * BK, row0, full);
          if (MODE == 0) {
            tma_load_2d(sB + 0 * B_ATOM_BYTES, &tmB0, n * 128, yb + kb * BK, full);
            tma_load_2d(sB + 1 * B_ATOM_BYTES, &tmB0, n * 128 + 64, yb + kb * BK, full);
            tma_load_2d(sB + 2 * B_ATOM_BYTES, &tmB1, n * 128, yb + kb * BK, full);
            tma_load_2d(sB + 3 * B_ATOM_BYTES, &tmB1, n * 128 + 64, yb + kb * BK, full);
          } else {
#pragma unroll
            for (int b = 0; b < BN / 64; ++b)
              tma_load_2d(sB + b * B_ATOM_BYTES, &tmB0, n * BN + b * 64, yb + kb * BK, full);
          }
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // make sure no load is still landing in shared memory when the CTA exits
      const int64_t first = issued > STAGES ? issued - STAGES : 0;
      for (int64_t j = first; j < issued; ++j)
        wait_drain(smem_u32(&bars[BAR_FULL + (j % STAGES)]), static_cast<uint32_t>((j / STAGES) & 1),
                   p.timeout_ns);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
        int row0, n, l;
        if (!tile_info(tile, row0, n, l)) continue;
        if (!wait_bounded(smem_u32(&bars[BAR_TEMPTY + acc]), acc_phase ^ 1u, wc)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!wait_bounded(smem_u32(&bars[BAR_FULL + stage]), phase, wc)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sA = smem_u32(smem + stage * STAGE_BYTES);
          const uint32_t sB = sA + A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / UMMA_K; ++kk) {
            // A: K-major, advance 16 bf16 = 32 bytes inside the swizzled row.
            // B: MN-major, advance 16 K-rows = two 8-row groups = 2048 bytes.
            const uint64_t a_desc = smem_desc_sw128(sA + kk * 32, 16, 1024);
            const uint64_t b_desc = smem_desc_sw128(sB + kk * 2048, B_ATOM_BYTES, 1024);
            tc_mma_f16(d_tmem, a_desc, b_desc, IDESC, (kb | kk) != 0 ? 1u : 0u);
          }
          tc_commit(smem_u32(&bars[BAR_EMPTY + stage]));
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(smem_u32(&bars[BAR_TFULL + acc]));
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      // all MMAs issued by this thread have completed once this arrives
      tc_commit(smem_u32(&bars[BAR_DRAIN]));
      wait_drain(smem_u32(&bars[BAR_DRAIN]), 0, p.timeout_ns);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue
    const int q = warp - 4;  // TMEM lane quarter this warp may access
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      int row0, n, l;
      if (!tile_info(tile, row0, n, l)) continue;
      if (!wait_bounded(smem_u32(&bars[BAR_TFULL + acc]), acc_phase, wc)) break;
      tc_fence_after();
      const int64_t row = row0 + q * 32 + lane;
      const uint32_t tbase =
          tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * BN);
      if (MODE == 0) {
        uint4* hrow = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p.out) +
                                               row * p.Nout + n * 128);
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t ra[32], rb[32];
          tmem_ld_32cols(tbase + c * 32, ra);
          tmem_ld_32cols(tbase + 128 + c * 32, rb);
          tmem_ld_wait();
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float h0 = silu(__uint_as_float(ra[2 * i])) * __uint_as_float(rb[2 * i]);
            const float h1 = silu(__uint_as_float(ra[2 * i + 1])) * __uint_as_float(rb[2 * i + 1]);
            pk[i] = pack_bf16x2(h0, h1);
          }
#pragma unroll
          for (int v = 0; v < 4; ++v)
            hrow[c * 4 + v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
        }
      } else {
        float4* yrow = reinterpret_cast<float4*>(reinterpret_cast<float*>(p.out) + row * p.Nout +
                                                 n * BN);
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t rv[32];
          tmem_ld_32cols(tbase + c * 32, rv);
          tmem_ld_wait();
#pragma unroll
          for (int v = 0; v < 8; ++v)
            yrow[c * 8 + v] = make_float4(__uint_as_float(rv[4 * v]), __uint_as_float(rv[4 * v + 1]),
                                          __uint_as_float(rv[4 * v + 2]),
                                          __uint_as_float(rv[4 * v + 3]));
        }
      }
      tc_fence_before();
      mbar_arrive(smem_u32(&bars[BAR_TEMPTY + acc]));
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
  }

  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// 2D bf16 tensor [outer, inner] (inner contiguous), box [box_outer, box_inner],
// 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
              uint32_t box_outer) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {inner * 2};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int MODE>
cudaError_t launch_mode(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                        const FfnParams& p, cudaStream_t s) {
  const size_t smem = smem_bytes_for(p.E);
  cudaError_t e = cudaFuncSetAttribute(ffn_gemm_kernel<MODE>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  ffn_gemm_kernel<MODE><<<device_sm_count(), NUM_THREADS, smem, s>>>(a, b0, b1, p);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_expert_ffn(const uint16_t* xg, const uint16_t* W1, const uint16_t* W3,
                              const uint16_t* W2, const int32_t* offsets, const int32_t* counts,
                              uint16_t* h, float* y, const moe_shape_t& sh, int64_t rows_max,
                              int32_t* dev_status, cudaStream_t s, cudaEvent_t ev_mid) {
  const int E = sh.E, H = sh.H, I = sh.I;
  CUtensorMap mA1, mW1, mW3, mA2, mW2;
  const uint64_t EH = static_cast<uint64_t>(E) * H, EI = static_cast<uint64_t>(E) * I;
  if (!make_map(&mA1, xg, H, rows_max, 64, BM) || !make_map(&mW1, W1, I, EH, 64, 64) ||
      !make_map(&mW3, W3, I, EH, 64, 64) || !make_map(&mA2, h, I, rows_max, 64, BM) ||
      !make_map(&mW2, W2, H, EI, 64, 64))
    return cudaErrorInvalidValue;
  FfnParams p1{offsets, counts, E, sh.P, H, I, rows_max, h, dev_status, kWaitTimeoutNs};
  cudaError_t e = launch_mode<0>(mA1, mW1, mW3, p1, s);
  if (e != cudaSuccess) return e;
  if (ev_mid) {
    e = cudaEventRecord(ev_mid, s);
    if (e != cudaSuccess) return e;
  }
  FfnParams p2{offsets, counts, E, sh.P, I, H, rows_max, y, dev_status, kWaitTimeoutNs};
  return launch_mode<1>(mA2, mW2, mW2, p2, s);
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
