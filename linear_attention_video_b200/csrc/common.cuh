// Shared definitions of the CUDA path (kernels and the C-ABI layer).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kda.h"

namespace kda {

// Problem description after host-side validation, with derived sizes.
struct Dims {
  int B, H, dk, dv;
  int64_t N, L;          // tokens per item, text prefix length
  int T, Hg, Wg;         // visual grid
  int text_k;
  int pt, ph, pw;        // 3D conv padding (tap offsets are a - pt etc.)
  int chunk;
  bool reuse_records;    // KDA_FLAG_REUSE_RECORDS: the workspace holds this problem's block records
  bool qkv_f16;          // KDA_FLAG_QKV_F16: convolved q', k', v' are fp16
};

// Device status word: the first uint32 of the workspace.
__device__ __forceinline__ void set_status(uint32_t* status, uint32_t code) {
  if (status) atomicCAS(status, 0u, code);
}

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Launchers (defined in the .cu files).
// out_f16: write fp16 outputs (the internal format the tensor-core scan reads) instead of dtype;
// out_f32: write fp32 outputs (what the backward pass recomputes).
cudaError_t launch_shortconv(const Dims& d, kda_dtype dt, const void* q, const void* k, const void* v,
                             const float* w_text, const float* w_vis, void* qo, void* ko, void* vo,
                             cudaStream_t s, int* launches, bool out_f16 = false, bool out_f32 = false);
// Backward of the visual conv: dx of the visual tokens (the transposed conv of dy,
// written as dtype) and dw_vis += the weight gradient (fp32, accumulated).
cudaError_t launch_shortconv_bwd_vis(const Dims& d, kda_dtype dt, const void* const x[3], const float* const dy[3],
                                     void* const dx[3], const float* w_vis, float* dw_vis, cudaStream_t s,
                                     int* launches);

// Backward pass (bwd.cu): gradients of kda_fwd.  Buffers as in kda_bwd (include/kda.h); ws holds
// bwd_workspace_bytes(d, dt) bytes, 256-byte aligned, its first word the status word.
size_t bwd_workspace_bytes(const Dims& d, kda_dtype dt);
cudaError_t launch_bwd(const Dims& d, kda_dtype dt, const void* q, const void* k, const void* v,
                       const float* log_alpha, const void* beta, const float* w_text, const float* w_vis,
                       const float* S0, const void* d_o, const float* dSN, void* dq, void* dk, void* dv,
                       float* dla, void* dbeta, float* dw_text, float* dw_vis, float* dS0, void* ws,
                       cudaStream_t s, int* launches);

cudaError_t launch_chunk_simt(const Dims& d, kda_dtype dt, const void* q, const void* k, const void* v,
                              const float* log_alpha, const void* beta, const float* S0, void* o,
                              float* SN, uint32_t* status, cudaStream_t s, int* launches);

size_t chunk_simt_smem_bytes(int dk, int chunk);

// tcgen05 path (bf16 problems with d_k = d_v = 128)
bool chunk_tc_supported(const Dims& d);
size_t chunk_tc_workspace_bytes(const Dims& d);
// fault (self-test of the bounded waits only): 1 = the record kernel's first CTA never issues its first
// input load, 2 = the state pass's first CTA never issues its first record load; wait_ns bounds every
// device wait of the two kernels.
constexpr uint64_t kWaitNs = 500000000ull;
cudaError_t launch_chunk_tc(const Dims& d, bool in_f16, const void* q, const void* k, const void* v,
                            const float* log_alpha, const void* beta, const float* S0, void* o, float* SN,
                            void* ws, uint32_t* status, cudaStream_t s, int* launches, int fault = 0,
                            uint64_t wait_ns = kWaitNs);

// Host-side validation (kda_api.cu), returning a kda_status.
int validate_problem(const kda_problem* p, kda_dtype dt, Dims* d);
int validate_scan_pointers(const void* q, const void* k, const void* v, const void* la, const void* beta, const void* o,
                           const void* s0, const void* sn);
// Records the launch count that kda_last_launch_count() reports for this host thread.
void set_last_launch_count(int launches);

}  // namespace kda
