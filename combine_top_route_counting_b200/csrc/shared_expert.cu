// The bf16 shared expert of the MXFP8 layer ("Mixture-of-Kittens: A MoE
// Megakernel for GB300 NVL72", section 5: beside the MXFP8 routed experts, a
// shared expert every token passes through runs in bf16). It is the routed
// FFN's arithmetic with one set of weights over all tokens, so it runs on the
// same persistent CTA-pair GEMMs (expert_ffn.cu) as a single expert whose
// segment is every token: a = x.Ws1, b = x.Ws3 (fp32 accumulation),
// hs = bf16(silu(a) * b), ys = hs.Ws2 (fp32). The layer's combine then starts
// each token's fixed-order sum from ys[t].
#include "internal.cuh"

namespace moe {
namespace {

// The one-segment table of the shared expert: rows [0, rows).
__global__ void one_segment_kernel(int32_t* off, int32_t rows) {
  off[0] = 0;
  off[1] = rows;
}

}  // namespace

cudaError_t launch_dense_ffn(const uint16_t* x, int64_t n_tokens, const uint16_t* Ws1,
                             const uint16_t* Ws3, const uint16_t* Ws2, uint16_t* xpad,
                             uint16_t* hs, float* ys, int32_t* off, int32_t H, int32_t I,
                             int32_t* dev_status, cudaStream_t s, int* counter) {
  if (n_tokens <= 0) return cudaSuccess;
  const int64_t rows = (n_tokens + 255) / 256 * 256;
  const size_t row_bytes = static_cast<size_t>(H) * 2;
  const uint16_t* a = x;
  cudaError_t e;
  if (rows != n_tokens) {  // the GEMM's tiles cover whole 256-row blocks: pad with zeros
    if (!xpad) return cudaErrorInvalidValue;
    if ((e = cudaMemcpyAsync(xpad, x, n_tokens * row_bytes, cudaMemcpyDeviceToDevice, s)) !=
        cudaSuccess)
      return e;
    if ((e = cudaMemsetAsync(xpad + n_tokens * H, 0, (rows - n_tokens) * row_bytes, s)) !=
        cudaSuccess)
      return e;
    a = xpad;
  }
  one_segment_kernel<<<1, 1, 0, s>>>(off, static_cast<int32_t>(rows));
  note_launches(1);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  moe_shape_t one{};
  one.P = 1;
  one.N = static_cast<int32_t>(n_tokens);
  one.E = 1;
  one.k = 1;
  one.H = H;
  one.I = I;
  one.pad = 256;
  return launch_expert_ffn(a, Ws1, Ws3, Ws2, off, nullptr, hs, ys, one, rows, dev_status, s,
                           nullptr, nullptr, counter);
}

}  // namespace moe
