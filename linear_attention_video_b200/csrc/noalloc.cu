// kda_chunk_fwd_noalloc: the chunked KDA scan for callers that cannot allocate
// device memory.
//
// Some callers run where cudaMalloc is unavailable or forbidden: code inside a
// custom allocator or memory-pool callback, inference runtimes that pre-plan
// every byte and reject allocations after start-up, or plugins handed only
// input and output buffers.  This variant of kda_chunk_fwd takes no workspace.
// Its scratch (the scan's per-block records and the device status word) lives
// in a file-scope __device__ array of kNoAllocScratchBytes, which every GPU that
// loads the library holds until the process exits.
//
// In host code the array's name is only a host-side stand-in, so the array's
// device address is obtained once per device, with that device current, through
// cudaGetSymbolAddress; the first call on a device does this, so make that first
// call before any stream capture.  Every call shares the array and it keeps the
// last call's contents: the status word is cleared at the start of each call,
// the records are fully rewritten.  Calls whose GPU work overlaps (different
// streams, or different host threads on one device) race on the array.  The
// cached address belongs to the device's primary context: after a
// cudaDeviceReset in the process it is stale, and this entry point must not be
// used again on that device.
#include <mutex>

#include "common.cuh"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;   // 64 MiB
constexpr size_t kStatusBytes = 256;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device (cached per device).
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KDA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_scratch_addr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return KDA_ERR_CUDA;
    g_scratch_addr[dev] = ptr;
  }
  *out = g_scratch_addr[dev];
  return KDA_OK;
}

}  // namespace

extern "C" int kda_chunk_fwd_noalloc(const kda_problem* p, kda_dtype dtype, const void* q, const void* k,
                                     const void* v, const float* log_alpha, const void* beta,
                                     const float* initial_state, void* o, float* final_state,
                                     uint32_t* device_status, void* stream) {
  kda::set_last_launch_count(0);
  kda::Dims d;
  int st = kda::validate_problem(p, dtype, &d);
  if (st) return st;
  if (d.reuse_records) return KDA_ERR_INVALID_ARG;   // the shared scratch keeps no records between calls
  if ((st = kda::validate_scan_pointers(q, k, v, log_alpha, beta, o, initial_state, final_state))) return st;
  if (device_status && (reinterpret_cast<uintptr_t>(device_status) & 3u)) return KDA_ERR_MISALIGNED;
  const bool tc = dtype == KDA_DT_BF16 && kda::chunk_tc_supported(d);
  const size_t need = kStatusBytes + (tc ? kda::chunk_tc_workspace_bytes(d) : 0);
  if (need > kNoAllocScratchBytes) return KDA_ERR_WORKSPACE;   // problem larger than the static scratch
  void* scratch = nullptr;
  if ((st = scratch_address(&scratch))) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t* status = device_status ? device_status : static_cast<uint32_t*>(scratch);
  if (cudaMemsetAsync(status, 0, sizeof(uint32_t), s) != cudaSuccess) return KDA_ERR_CUDA;
  int launches = 0;
  cudaError_t e = cudaSuccess;
  if (d.N == 0) {
    if (final_state) {
      const size_t bytes = (size_t)d.B * d.H * d.dk * d.dv * sizeof(float);
      e = initial_state ? cudaMemcpyAsync(final_state, initial_state, bytes, cudaMemcpyDeviceToDevice, s)
                        : cudaMemsetAsync(final_state, 0, bytes, s);
    }
  } else if (tc) {
    e = kda::launch_chunk_tc(d, d.qkv_f16, q, k, v, log_alpha, beta, initial_state, o, final_state,
                             static_cast<char*>(scratch) + kStatusBytes, status, s, &launches);
  } else {
    e = kda::launch_chunk_simt(d, dtype, q, k, v, log_alpha, beta, initial_state, o, final_state, status, s,
                               &launches);
  }
  if (e != cudaSuccess) return KDA_ERR_CUDA;
  kda::set_last_launch_count(launches);
  return KDA_OK;
}
