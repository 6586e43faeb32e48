// Internal launchers shared by the C-ABI layer (api.cu) and the kernel files.
#pragma once

#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "moe.h"

namespace moe {

// Kernels launched by this library in this process (moe_launch_count).
void note_launches(int64_t n);

// The shape limits every entry point checks (include/moe.h): MOE_OK,
// MOE_INVALID_ARG (null shape) or MOE_UNSUPPORTED_SHAPE.
moe_status_t check_shape(const moe_shape_t* s);
// Pointer on a 16-byte boundary (null passes).
bool aligned16(const void* p);

// Number of SMs of the current device (cached per device).
int device_sm_count();

// A token slice [t0, t0+Tm) of every peer: the unit the schedule, dispatch,
// FFN and combine work on (the whole input is t0 = 0, Tm = N).
struct Slice {
  int32_t t0, Tm;
};

// Words of device scratch that a call's later kernels expect to find zero
// (the GEMMs' tile counter and landing flags, the schedule's grid barrier):
// the routing kernel, the first kernel of a layer call, zeroes them in its
// first block, so the layer needs no memset of its own.
struct ZeroSpec {
  int* a;
  int32_t na;
  int* b;
  int32_t nb;
};

// Step 1 (z, if not null: words to zero, as above)
cudaError_t launch_route_topk(const float* logits, int32_t* ids, float* gates, int64_t n_tokens,
                              int32_t E, int32_t k, cudaStream_t s, const ZeroSpec* z = nullptr);

// Step 2
constexpr int kSchedBlockRoutes = 2048;  // routes per counting block (8 warps x 256)
size_t schedule_ws_bytes(int32_t P, int32_t N, int32_t k, int32_t E);
// barrier_zeroed: the schedule_zero_words(sh) words of ws from
// schedule_barrier_word on (the grid barrier and the totals its one-launch
// kernel accumulates) are already zero (else the launch zeroes them first).
cudaError_t launch_schedule(const int32_t* ids, const moe_shape_t& sh, Slice sl, int32_t* phi,
                            int32_t* offsets, int32_t* counts, int32_t* route_row, int32_t* ws,
                            int32_t* dev_status, cudaStream_t s, bool barrier_zeroed = false);
// The word of the schedule's scratch that its one-launch kernel's grid
// barrier counts on (after the [P][blocks][E] counters of the whole batch).
int32_t* schedule_barrier_word(int32_t* ws, const moe_shape_t& sh);
int32_t schedule_zero_words(const moe_shape_t& sh);

// The schedule's one-launch kernel with a grid barrier that waits for one
// block more than the launch has: every block gives up after timeout_ns and
// raises MOE_DEV_TIMEOUT (failure-detection self test). cudaErrorInvalidConfiguration
// if the shape does not take the one-launch kernel.
cudaError_t launch_schedule_barrier_selftest(const int32_t* ids, const moe_shape_t& sh,
                                             int32_t* phi, int32_t* offsets, int32_t* counts,
                                             int32_t* route_row, int32_t* ws, int32_t* dev_status,
                                             int64_t timeout_ns, cudaStream_t s);

// Step 3a
cudaError_t launch_dispatch(const uint16_t* x, const int32_t* phi, const int32_t* offsets,
                            uint16_t* xg, const moe_shape_t& sh, int64_t rows_max,
                            int32_t* dev_status, cudaStream_t s);

// The persistent GEMMs below take their tiles from a tile counter: two device
// int32 words {next tile, CTAs finished} that are zero when a launch starts
// and that the launch's last CTA puts back to zero. `counter` is the caller's
// (the layer entry points keep one in their workspace, zeroed once per call;
// launches on one stream reuse it one after another), or null: a slot of the
// device's pool (tile_counter_for_current_device).

// The pull dispatch fused into GEMM1 (steps 3a + 3b in one kernel): GEMM1's
// spare warp lands the rows x[Phi[row]] into xg block by block while the
// tensor cores work on blocks already landed. next (one int32) and ready
// ([rows_max / 128] int32) are device scratch the caller zeroes before the
// launch.
struct LandArgs {
  const uint16_t* x;    // token activations [P*N, H]
  const int32_t* phi;   // [rows_max, 2]
  int* next;
  int* ready;
};

// Step 3b (two kernels; ev_mid, if not null, is recorded between them).
// ab (training, pair tiles only): also keep the bf16 pre-activations [a | b].
// land (pair tiles only): GEMM1 also performs the dispatch into xg.
cudaError_t launch_expert_ffn(const uint16_t* xg, const uint16_t* W1, const uint16_t* W3,
                              const uint16_t* W2, const int32_t* offsets, const int32_t* counts,
                              uint16_t* h, float* y, const moe_shape_t& sh, int64_t rows_max,
                              int32_t* dev_status, cudaStream_t s, cudaEvent_t ev_mid,
                              uint16_t* ab = nullptr, int* counter = nullptr,
                              const LandArgs* land = nullptr);

// Steps 3a+3b fused: GEMM1 pulls its A rows from x by Phi (no xg buffer)
cudaError_t launch_expert_ffn_gather(const uint16_t* x, const int32_t* phi, const uint16_t* W1,
                                     const uint16_t* W3, const uint16_t* W2,
                                     const int32_t* offsets, const int32_t* counts, uint16_t* h,
                                     float* y, const moe_shape_t& sh, int64_t rows_max,
                                     int32_t* dev_status, cudaStream_t s, cudaEvent_t ev_mid);

// Step 4. shared (optional, fp32 [P*N rows, H]): the shared expert's output,
// the start of each token's fixed-order sum.
cudaError_t launch_combine(const float* y, const int32_t* route_row, const float* gates,
                           uint16_t* out, const moe_shape_t& sh, Slice sl, int64_t rows_max,
                           int32_t* dev_status, cudaStream_t s, const float* shared = nullptr);

// The bf16 shared expert: the SwiGLU FFN of every token x[t] (t < n_tokens)
// with one set of weights Ws1, Ws3 [H, I], Ws2 [I, H], run as the one segment
// of launch_expert_ffn over round_up(n_tokens, 256) rows. hs bf16 and ys fp32
// have that many rows. xpad ([rows, H] bf16) takes a zero-padded copy of x
// when n_tokens is not a multiple of 256 (else x is read in place and xpad
// may be null); off: device int32[2] scratch for the one-segment table.
cudaError_t launch_dense_ffn(const uint16_t* x, int64_t n_tokens, const uint16_t* Ws1,
                             const uint16_t* Ws3, const uint16_t* Ws2, uint16_t* xpad,
                             uint16_t* hs, float* ys, int32_t* off, int32_t H, int32_t I,
                             int32_t* dev_status, cudaStream_t s, int* counter = nullptr);

// 2D tensor map over [outer, inner] (inner contiguous) bf16 (or fp32)
// elements with box [box_outer, box_inner] and 128-byte swizzle (64-byte with
// swizzle64); false if the driver entry point is missing or rejects the
// arguments.
bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
              uint32_t box_outer, bool fp32 = false, bool swizzle64 = false);

// A tile counter for one launch of a persistent GEMM on the current device:
// the next slot of a per-device pool of 256 (round robin). A slot is clean
// again as soon as the launch that used it has finished, so two launches
// share one only if both run at the same moment while 255 other pool launches
// were enqueued between them (or one captured graph is replayed on two
// streams at once).
cudaError_t tile_counter_for_current_device(int** out);

// ---------------------------------------------------------------- backward
// Pull-reverse-combine: dys[row] = dout[Phi[row]], gate_row[row] = the gate of
// the row's route (padding rows: zeros).
cudaError_t launch_reverse_combine(const uint16_t* dout, const int32_t* phi,
                                   const int32_t* offsets, const int32_t* route_row,
                                   const float* gates, uint16_t* dys, float* gate_row,
                                   const moe_shape_t& sh, int64_t rows_max, int32_t* dev_status,
                                   cudaStream_t s);

// Expert FFN activation gradients (two kernels; ev_mid recorded between them).
cudaError_t launch_expert_ffn_dgrad(const uint16_t* dys, const float* gate_row, const uint16_t* ab,
                                    const uint16_t* h, const uint16_t* W1, const uint16_t* W3,
                                    const uint16_t* W2, const int32_t* offsets,
                                    const int32_t* counts, uint16_t* dab, uint16_t* hg,
                                    float* part, float* dxg, const moe_shape_t& sh,
                                    int64_t rows_max, int32_t* dev_status, cudaStream_t s,
                                    cudaEvent_t ev_mid, int* counter = nullptr);

// Push-reverse-dispatch: dx[t] = bf16(sum_j dxg[route_row[t, j]]), ascending j.
cudaError_t launch_reverse_dispatch(const float* dxg, const int32_t* route_row, uint16_t* dx,
                                    const moe_shape_t& sh, int64_t rows_max, int32_t* dev_status,
                                    cudaStream_t s);

// Router gradient from the gate-gradient partial sums [rows, npart].
cudaError_t launch_router_backward(const float* part, int32_t npart, const int32_t* route_row,
                                   const int32_t* ids, const float* gates, float* dlogits,
                                   int64_t n_tokens, int32_t E, int32_t k, int64_t rows_max,
                                   int32_t* dev_status, cudaStream_t s);

// Expert weight gradients (two kernels: dW2, then dW1 | dW3).
cudaError_t launch_expert_ffn_wgrad(const uint16_t* xg, const uint16_t* dys, const uint16_t* dab,
                                    const uint16_t* hg, const int32_t* offsets,
                                    const int32_t* counts, float* dW1, float* dW3, float* dW2,
                                    const moe_shape_t& sh, int64_t rows_max, int32_t* dev_status,
                                    cudaStream_t s, cudaEvent_t ev_mid, int* counter = nullptr);

// ---------------------------------------------------------------- MXFP8
// MX quantisation (E4M3 codes, one E8M0 scale per 32 values along the row).
cudaError_t launch_mx_quantize_rows(const uint16_t* src, int64_t n_rows, int32_t K, uint8_t* q,
                                    uint8_t* scale, cudaStream_t s);
// The pull dispatch with the MX quantisation fused: xq/xs rows of the gathered tokens.
// tiled: the scales in the tensor-core layout (mx_tiled_offset) instead of row-major.
cudaError_t launch_dispatch_mxfp8(const uint16_t* x, const int32_t* phi, const int32_t* offsets,
                                  uint8_t* xq, uint8_t* xs, const moe_shape_t& sh,
                                  int64_t rows_max, int32_t* dev_status, cudaStream_t s,
                                  bool tiled = false);

// Byte offset of the E8M0 scale of row r, 32-value block b, in the tiled
// layout of a [R, K] code matrix (R and K multiples of 128): 512-byte atoms
// of 128 rows x 4 blocks, K-atoms of a row block consecutive; inside an atom
// row r at (r % 32) * 16 + ((r / 32) % 4) * 4, block b at b % 4 -- the layout
// tcgen05.cp (32x128b, warpx4) moves into TMEM for the block-scaled MMA.
__host__ __device__ __forceinline__ int64_t mx_tiled_offset(int64_t r, int32_t b, int32_t kblocks) {
  return ((r >> 7) * (kblocks >> 2) + (b >> 2)) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (b & 3);
}

// Expert weights to MXFP8 for the block-scaled GEMMs: W bf16 [E, K, N] ->
// codes [E, N, K] (transposed: K-major) and tiled scales over the [E*N, K/32]
// table. K % 128 == 0, N % 128 == 0.
cudaError_t launch_mx_quantize_weights(const uint16_t* W, int32_t E, int32_t K, int32_t N,
                                       uint8_t* q, uint8_t* scale, cudaStream_t s);

// The grouped SwiGLU expert FFN on MXFP8 operands (block-scaled tcgen05, CTA
// pairs): GEMM1 + SwiGLU + MX quantisation of h, then GEMM2 -> fp32 y.
// ev_mid, if not null, is recorded between the two kernels. land (if not
// null): GEMM1 quantises x[Phi[row]] into xq, xs (tiled scales) itself, block
// by block, instead of reading a dispatch's output; its flags must be zero.
cudaError_t launch_expert_ffn_mxfp8(const uint8_t* xq, const uint8_t* xs, const uint8_t* W1q,
                                    const uint8_t* W1s, const uint8_t* W3q, const uint8_t* W3s,
                                    const uint8_t* W2q, const uint8_t* W2s,
                                    const int32_t* offsets, const int32_t* counts, uint8_t* hq,
                                    uint8_t* hs, float* y, const moe_shape_t& sh,
                                    int64_t rows_max, int32_t* dev_status, cudaStream_t s,
                                    cudaEvent_t ev_mid, int* counter = nullptr,
                                    const LandArgs* land = nullptr);

// 2D tensor map over a [outer, inner] uint8 matrix, box [box_outer, box_inner],
// 128-byte swizzle.
bool make_map_u8(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
                 uint32_t box_inner, uint32_t box_outer);
// Tensor map whose box is one 512-byte scale atom of a tiled scale table.
bool make_map_sf_atoms(CUtensorMap* m, const void* base, uint64_t n_atoms);

// Failure-detection self test (bounded wait on an mbarrier nothing completes).
cudaError_t launch_selftest_wait(int32_t* dev_status, int64_t timeout_ns, cudaStream_t s);

// Default limit of every bounded device wait.
constexpr int64_t kWaitTimeoutNs = 1000000000ll;

}  // namespace moe
