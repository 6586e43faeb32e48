// MXFP8 quantisation of bf16 rows, alone or fused into the pull dispatch
// ("Mixture-of-Kittens: A MoE Megakernel for GB300 NVL72", section 5: MXFP8
// routed experts with the quantisation fused into the dispatch; the OCP
// Microscaling formats, MXFP8 with E4M3 elements).
//
// Each block of 32 consecutive values of a row is quantised by the rule in
// mx_block.cuh (one E8M0 scale, 32 E4M3 codes).
//
// One warp per row; lane j quantises blocks j, j+32, ...: its 64 input bytes
// and 32 output bytes are contiguous with its neighbours', so every load and
// store of the warp is coalesced. HBM-bound: 2 bytes read and 1 + 1/32 bytes
// written per element.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "internal.cuh"
#include "mx_block.cuh"

namespace moe {
namespace {

using mx::mx_block;

// GATHER: row r of the output comes from token phi[r] of x (pad rows: zeros,
// scale code 0); otherwise row r of src. TILED: scales in the tensor-core
// layout (mx_tiled_offset), else row-major [rows, K/32].
template <bool GATHER, bool TILED = false>
__global__ void __launch_bounds__(256) mx_rows_kernel(const uint4* __restrict__ src,
                                                      const int2* __restrict__ phi,
                                                      const int32_t* __restrict__ offsets,
                                                      uint4* __restrict__ q, uint8_t* __restrict__ sc,
                                                      int64_t n_rows, int K, int P, int N, int E,
                                                      int64_t rows_max, int32_t* dev_status) {
  int64_t rows = n_rows;
  if (GATHER) {
    rows = __ldg(offsets + E);
    if (rows < 0 || rows > rows_max) {
      if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(dev_status, MOE_DEV_BAD_SCHEDULE);
      return;
    }
  }
  const int lane = threadIdx.x & 31;
  const int nblk = K / 32;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * 8;
  int bad = 0;
  for (int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5); row < rows;
       row += nwarps) {
    int64_t srow = row;
    bool zero = false;
    if (GATHER) {
      const int2 e = __ldg(phi + row);
      const bool ok = e.x >= 0 && e.x < P && e.y >= 0 && e.y < N;
      if (!ok && (e.x >= 0 || e.y != -1)) bad = 1;  // (-1,-1) is padding
      zero = !ok;
      srow = ok ? static_cast<int64_t>(e.x) * N + e.y : 0;
    }
    const uint4* s = src + srow * (K / 8);
    uint4* qrow = q + row * (K / 16);
    uint8_t* srow_sc = sc + row * nblk;
    for (int b = lane; b < nblk; b += 32) {
      uint4 in[4];
#pragma unroll
      for (int v = 0; v < 4; ++v) in[v] = zero ? make_uint4(0, 0, 0, 0) : __ldg(s + b * 4 + v);
      uint4 out[2];
      uint8_t scale;
      mx_block(in, out, scale);
      qrow[b * 2] = out[0];
      qrow[b * 2 + 1] = out[1];
      if (TILED) sc[mx_tiled_offset(row, b, nblk)] = scale;
      else srow_sc[b] = scale;
    }
  }
  if (bad) atomicOr(dev_status, MOE_DEV_BAD_SCHEDULE);
}

// Expert weights W [E, K, N] (bf16, N contiguous) to K-major MXFP8: codes
// q [E, N, K] and tiled scales of the [E*N, K/32] table, blocks of 32 along K.
// One block per (expert, 128 K-rows, 64 columns): the tile is staged in
// shared memory with coalesced 16-byte loads; thread t then quantises column
// t % 64, K block t / 64 (a warp reads one shared row of 64 contiguous bytes
// per step) and writes its 32 codes as two 16-byte stores.
__global__ void __launch_bounds__(256) mx_weights_kernel(const uint4* __restrict__ W,
                                                         uint8_t* __restrict__ q,
                                                         uint8_t* __restrict__ sc, int K, int N) {
  __shared__ __align__(16) uint16_t tile[128 * 64];
  const int tiles_n = N / 64, tiles_k = K / 128;
  const int64_t bid = blockIdx.x;
  const int nt = static_cast<int>(bid % tiles_n);
  const int kt = static_cast<int>((bid / tiles_n) % tiles_k);
  const int64_t e = bid / (static_cast<int64_t>(tiles_n) * tiles_k);
  const int t = threadIdx.x;
#pragma unroll
  for (int i = 0; i < 4; ++i) {  // 1,024 16-byte chunks: row idx / 8, chunk idx % 8
    const int idx = t + 256 * i;
    const int r = idx >> 3, c8 = idx & 7;
    const int64_t src = ((e * K + static_cast<int64_t>(kt) * 128 + r) * N + nt * 64) / 8 + c8;
    reinterpret_cast<uint4*>(tile)[r * 8 + c8] = __ldg(W + src);
  }
  __syncthreads();
  const int n = t & 63, j = t >> 6;
  uint4 in[4];
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int k0 = j * 32 + v * 8 + 2 * i;  // elements k0 (low half) and k0 + 1
      w[i] = static_cast<uint32_t>(tile[k0 * 64 + n]) |
             (static_cast<uint32_t>(tile[(k0 + 1) * 64 + n]) << 16);
    }
    in[v] = make_uint4(w[0], w[1], w[2], w[3]);
  }
  uint4 out[2];
  uint8_t scale;
  mx_block(in, out, scale);
  const int64_t row = e * N + nt * 64 + n;  // row of the transposed matrix
  const int b = kt * 4 + j;                 // 32-block along K
  uint4* qrow = reinterpret_cast<uint4*>(q + row * K + static_cast<int64_t>(b) * 32);
  qrow[0] = out[0];
  qrow[1] = out[1];
  sc[mx_tiled_offset(row, b, K / 32)] = scale;
}

int grid_for(int64_t rows) {
  const int64_t want = (rows + 7) / 8;
  const int64_t cap = static_cast<int64_t>(device_sm_count()) * 8;
  return static_cast<int>(want < cap ? want : cap);
}

}  // namespace

cudaError_t launch_mx_quantize_rows(const uint16_t* src, int64_t n_rows, int32_t K, uint8_t* q,
                                    uint8_t* scale, cudaStream_t s) {
  if (n_rows <= 0) return cudaSuccess;
  mx_rows_kernel<false><<<grid_for(n_rows), 256, 0, s>>>(
      reinterpret_cast<const uint4*>(src), nullptr, nullptr, reinterpret_cast<uint4*>(q), scale,
      n_rows, K, 0, 0, 0, 0, nullptr);
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_dispatch_mxfp8(const uint16_t* x, const int32_t* phi, const int32_t* offsets,
                                  uint8_t* xq, uint8_t* xs, const moe_shape_t& sh,
                                  int64_t rows_max, int32_t* dev_status, cudaStream_t s,
                                  bool tiled) {
  if (rows_max <= 0) return cudaSuccess;
  auto kernel = tiled ? mx_rows_kernel<true, true> : mx_rows_kernel<true, false>;
  kernel<<<grid_for(rows_max), 256, 0, s>>>(
      reinterpret_cast<const uint4*>(x), reinterpret_cast<const int2*>(phi), offsets,
      reinterpret_cast<uint4*>(xq), xs, rows_max, sh.H, sh.P, sh.N, sh.E, rows_max, dev_status);
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_mx_quantize_weights(const uint16_t* W, int32_t E, int32_t K, int32_t N,
                                       uint8_t* q, uint8_t* scale, cudaStream_t s) {
  const int64_t blocks = static_cast<int64_t>(E) * (K / 128) * (N / 64);
  if (blocks <= 0) return cudaSuccess;
  mx_weights_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(
      reinterpret_cast<const uint4*>(W), q, scale, K, N);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace moe
