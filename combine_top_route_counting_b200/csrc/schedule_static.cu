// moe_schedule_static_ws: the schedule with its scratch in a fixed device array.
//
// Some callers cannot hand this library a scratch buffer: a plugin that a host
// application calls with nothing but its input and output buffers, or a
// serving loop that forbids cudaMalloc on its hot path because an allocation
// can synchronise the device and stall every other stream. For them this file
// keeps the schedule's per-block counters in a file-scope device array that
// is part of the loaded library, so the call itself allocates nothing.
//
// The array is a host-side stand-in in host code: its device address is
// fetched with cudaGetSymbolAddress once per device (the first call made with
// that device current) and passed to the kernels like any other pointer.
#include <mutex>

#include "internal.cuh"

namespace moe {
namespace {

// 1,048,576 int32 words (4 MiB), held by every GPU that loads the library.
// Enough for P * ceil(N*k / 2048) * E up to that count, e.g. 8 peers x 65,536
// tokens x top-8 with 384 experts.
constexpr int64_t kStaticSchedWords = int64_t{1} << 20;
static __device__ __align__(256) int32_t g_sched_scratch[kStaticSchedWords];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
int32_t* g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of g_sched_scratch on the current device (set up once per device).
cudaError_t scratch_for_current_device(int32_t** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_sched_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = static_cast<int32_t*>(p);
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" moe_status_t moe_schedule_static_ws(const int32_t* ids, int32_t* phi, int32_t* offsets,
                                               int32_t* counts, int32_t* route_row,
                                               int32_t* dev_status, const moe_shape_t* shape,
                                               void* stream) {
  // the same argument checks as moe_schedule
  const moe_status_t st = check_shape(shape);
  if (st != MOE_OK) return st;
  const moe_shape_t& s = *shape;
  if (!phi || !offsets || !counts || !dev_status) return MOE_INVALID_ARG;
  if (s.N > 0 && (!ids || !route_row)) return MOE_INVALID_ARG;
  if (!aligned16(ids) || !aligned16(phi) || !aligned16(route_row)) return MOE_INVALID_ARG;
  // the same counter layout moe_schedule uses: [P][ceil(N*k/2048)][E] int32
  if (schedule_ws_bytes(s.P, s.N, s.k, s.E) > static_cast<size_t>(kStaticSchedWords) * 4)
    return MOE_WORKSPACE_TOO_SMALL;
  int32_t* scratch = nullptr;
  if (scratch_for_current_device(&scratch) != cudaSuccess) return MOE_CUDA_ERROR;
  // The counters need no clearing: the count kernel writes every word the
  // scan and scatter kernels read before they read it.
  const cudaError_t e = launch_schedule(ids, s, Slice{0, s.N}, phi, offsets, counts, route_row,
                                        scratch, dev_status, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MOE_OK : MOE_CUDA_ERROR;
}
