// Host-side helpers shared by the persistent GEMM launchers: TMA tensor maps
// and the per-launch tile counters.
#include <mutex>

#include "internal.cuh"

namespace moe {

// Tile counters the scheduler threads of the persistent GEMMs take tile ids
// from, for launches whose caller passes none: {next tile, CTAs finished}
// per slot, zero at load time and put back to zero by the last CTA of each
// launch. Each launch takes the next slot (round robin); nothing is written
// to a slot when a launch is enqueued, so a launch waiting in one stream is
// never disturbed by launches enqueued on others.
constexpr int kTileCounterSlots = 256;
__device__ int g_tile_counter[kTileCounterSlots * 2];

namespace {
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

}  // namespace

bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
              uint32_t box_outer, bool fp32, bool swizzle64) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {inner * (fp32 ? 4 : 2)};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, fp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
            const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            swizzle64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_map_u8(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
                 uint32_t box_inner, uint32_t box_outer) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {inner};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_map_sf_atoms(CUtensorMap* m, const void* base, uint64_t n_atoms) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {128, n_atoms};  // 128 words of 4 scale bytes per atom
  const cuuint64_t strides[1] = {512};
  const cuuint32_t box[2] = {128, 1};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t tile_counter_for_current_device(int** out) {
  static std::mutex mu;
  static int* ptrs[64] = {nullptr};
  static uint32_t next[64] = {0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (!ptrs[dev]) {
    void* ptr = nullptr;
    if ((e = cudaGetSymbolAddress(&ptr, g_tile_counter)) != cudaSuccess) return e;
    ptrs[dev] = static_cast<int*>(ptr);
  }
  *out = ptrs[dev] + 2 * (next[dev]++ % kTileCounterSlots);
  return cudaSuccess;
}

}  // namespace moe
