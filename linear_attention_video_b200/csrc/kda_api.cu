// C-ABI layer: argument validation, workspace layout, dispatch to the kernels.
// The operations and layouts are documented in include/kda.h.
#include <string.h>

#include "common.cuh"

namespace {

thread_local int g_last_launches = 0;

constexpr size_t kStatusBytes = 256;

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
inline size_t elem_size(kda_dtype dt) { return dt == KDA_DT_BF16 ? 2 : 4; }

// Validates the problem and fills `d`.  Returns a kda_status.
int make_dims(const kda_problem* p, kda_dtype dt, kda::Dims* d) {
  if (!p) return KDA_ERR_INVALID_ARG;
  if (dt != KDA_DT_BF16 && dt != KDA_DT_F32) return KDA_ERR_INVALID_ARG;
  if (p->B < 1 || p->H < 1 || p->dk < 1 || p->dv < 1) return KDA_ERR_INVALID_ARG;
  if (p->text_len < 0 || p->grid_t < 0 || p->grid_h < 0 || p->grid_w < 0) return KDA_ERR_INVALID_ARG;
  const bool any_grid = p->grid_t || p->grid_h || p->grid_w;
  const bool all_grid = p->grid_t && p->grid_h && p->grid_w;
  if (any_grid && !all_grid) return KDA_ERR_INVALID_ARG;
  if (p->text_k < 1 || p->vis_kt < 1 || p->vis_kh < 1 || p->vis_kw < 1 || p->chunk < 1)
    return KDA_ERR_INVALID_ARG;
  if (p->flags & ~(KDA_FLAG_VIS_CAUSAL_T | KDA_FLAG_REUSE_RECORDS | KDA_FLAG_QKV_F16)) return KDA_ERR_INVALID_ARG;
  if (p->dk != p->dv || (p->dk != 64 && p->dk != 128)) return KDA_ERR_UNSUPPORTED;
  if (p->text_k > 8) return KDA_ERR_UNSUPPORTED;
  if (p->vis_kt != 3 || p->vis_kh != 3 || p->vis_kw != 3) return KDA_ERR_UNSUPPORTED;
  if (p->chunk != 16 && p->chunk != 32 && p->chunk != 64) return KDA_ERR_UNSUPPORTED;
  const int64_t vis = (int64_t)p->grid_t * p->grid_h * p->grid_w;
  const int64_t N = p->text_len + vis;
  // keep every element index well inside int64 and grid dims inside CUDA limits
  if (N > (int64_t(1) << 31) || (int64_t)p->B * N * p->H * p->dk > (int64_t(1) << 40))
    return KDA_ERR_UNSUPPORTED;
  // the 3D conv indexes one frame (grid_h * grid_w tokens x all channels) with 32-bit offsets
  if ((int64_t)p->grid_h * p->grid_w * p->H * p->dk >= (int64_t(1) << 31)) return KDA_ERR_UNSUPPORTED;
  d->B = p->B; d->H = p->H; d->dk = p->dk; d->dv = p->dv;
  d->N = N; d->L = p->text_len;
  d->T = p->grid_t; d->Hg = p->grid_h; d->Wg = p->grid_w;
  d->text_k = p->text_k;
  d->pt = (p->flags & KDA_FLAG_VIS_CAUSAL_T) ? p->vis_kt - 1 : (p->vis_kt - 1) / 2;
  d->ph = (p->vis_kh - 1) / 2;
  d->pw = (p->vis_kw - 1) / 2;
  d->chunk = p->chunk;
  d->reuse_records = (p->flags & KDA_FLAG_REUSE_RECORDS) != 0;
  d->qkv_f16 = (p->flags & KDA_FLAG_QKV_F16) != 0;
  // fp16 activations exist only where the tensor-core scan reads them (bf16, d = 128)
  if (d->qkv_f16 && !(dt == KDA_DT_BF16 && kda::chunk_tc_supported(*d))) return KDA_ERR_UNSUPPORTED;
  return KDA_OK;
}

size_t act_bytes(const kda::Dims& d, kda_dtype dt) {
  return (size_t)d.B * d.N * d.H * d.dk * elem_size(dt);
}

bool use_tc(const kda::Dims& d, kda_dtype dt) { return dt == KDA_DT_BF16 && kda::chunk_tc_supported(d); }

// status word | q', k', v' (conv outputs) | tensor-core scan records
size_t workspace_bytes(const kda::Dims& d, kda_dtype dt) {
  size_t n = kStatusBytes + 3 * align256(act_bytes(d, dt));
  if (use_tc(d, dt)) n += align256(kda::chunk_tc_workspace_bytes(d));
  return n;
}

size_t tc_records_offset(const kda::Dims& d, kda_dtype dt) { return kStatusBytes + 3 * align256(act_bytes(d, dt)); }

int cuda_status(cudaError_t e) { return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA; }

int check_ptrs(std::initializer_list<const void*> required, std::initializer_list<const void*> optional) {
  for (const void* p : required) {
    if (!p) return KDA_ERR_INVALID_ARG;
    if (!aligned16(p)) return KDA_ERR_MISALIGNED;
  }
  for (const void* p : optional)
    if (p && !aligned16(p)) return KDA_ERR_MISALIGNED;
  return KDA_OK;
}

int check_workspace(const kda::Dims& d, kda_dtype dt, void* ws, size_t ws_bytes) {
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u)) return KDA_ERR_WORKSPACE;
  if (ws_bytes < workspace_bytes(d, dt)) return KDA_ERR_WORKSPACE;
  return KDA_OK;
}

// The scan itself; the workspace status word has been cleared by the caller.
// in_f16: q', k', v' are the internal fp16 conv outputs (tensor-core path only).
int run_scan(const kda::Dims& d, kda_dtype dt, const void* q, const void* k, const void* v,
             const float* la, const void* beta, const float* S0, void* o, float* SN,
             void* workspace, cudaStream_t s, int* launches, bool in_f16) {
  uint32_t* status = static_cast<uint32_t*>(workspace);
  if (d.N == 0) {
    if (SN) {
      const size_t bytes = (size_t)d.B * d.H * d.dk * d.dv * sizeof(float);
      cudaError_t e = S0 ? cudaMemcpyAsync(SN, S0, bytes, cudaMemcpyDeviceToDevice, s)
                         : cudaMemsetAsync(SN, 0, bytes, s);
      return cuda_status(e);
    }
    return KDA_OK;
  }
  if (use_tc(d, dt)) {
    void* rec = static_cast<char*>(workspace) + tc_records_offset(d, dt);
    return cuda_status(kda::launch_chunk_tc(d, in_f16, q, k, v, la, beta, S0, o, SN, rec, status, s, launches));
  }
  return cuda_status(kda::launch_chunk_simt(d, dt, q, k, v, la, beta, S0, o, SN, status, s, launches));
}

}  // namespace

namespace kda {
// Validation shared with the allocation-free entry point (noalloc.cu).
int validate_problem(const kda_problem* p, kda_dtype dt, Dims* d) { return make_dims(p, dt, d); }
int validate_scan_pointers(const void* q, const void* k, const void* v, const void* la, const void* beta, const void* o,
                           const void* s0, const void* sn) {
  return check_ptrs({q, k, v, la, beta, o}, {s0, sn});
}
}  // namespace kda

extern "C" {

int64_t kda_tokens(const kda_problem* p) {
  if (!p || p->text_len < 0 || p->grid_t < 0 || p->grid_h < 0 || p->grid_w < 0) return -1;
  const bool any_grid = p->grid_t || p->grid_h || p->grid_w;
  const bool all_grid = p->grid_t && p->grid_h && p->grid_w;
  if (any_grid && !all_grid) return -1;
  return p->text_len + (int64_t)p->grid_t * p->grid_h * p->grid_w;
}

size_t kda_workspace_bytes(const kda_problem* p, kda_dtype dtype) {
  kda::Dims d;
  if (make_dims(p, dtype, &d) != KDA_OK) return 0;
  return workspace_bytes(d, dtype);
}

int kda_shortconv_fwd(const kda_problem* p, kda_dtype dtype, const void* q, const void* k,
                      const void* v, const float* w_text, const float* w_vis, void* q_out,
                      void* k_out, void* v_out, void* stream) {
  g_last_launches = 0;
  kda::Dims d;
  int st = make_dims(p, dtype, &d);
  if (st) return st;
  if (d.reuse_records) return KDA_ERR_INVALID_ARG;
  if ((st = check_ptrs({q, k, v, w_text, w_vis, q_out, k_out, v_out}, {}))) return st;
  int launches = 0;
  st = cuda_status(kda::launch_shortconv(d, dtype, q, k, v, w_text, w_vis, q_out, k_out, v_out,
                                         static_cast<cudaStream_t>(stream), &launches, d.qkv_f16));
  if (!st) g_last_launches = launches;
  return st;
}

int kda_chunk_fwd(const kda_problem* p, kda_dtype dtype, const void* q, const void* k, const void* v,
                  const float* log_alpha, const void* beta, const float* initial_state, void* o,
                  float* final_state, void* workspace, size_t workspace_bytes_, void* stream) {
  g_last_launches = 0;
  kda::Dims d;
  int st = make_dims(p, dtype, &d);
  if (st) return st;
  if ((st = check_ptrs({q, k, v, log_alpha, beta, o}, {initial_state, final_state}))) return st;
  if ((st = check_workspace(d, dtype, workspace, workspace_bytes_))) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t* status = static_cast<uint32_t*>(workspace);
  if ((st = cuda_status(cudaMemsetAsync(status, 0, sizeof(uint32_t), s)))) return st;
  int launches = 0;
  st = run_scan(d, dtype, q, k, v, log_alpha, beta, initial_state, o, final_state, workspace, s, &launches,
                d.qkv_f16);
  if (!st) g_last_launches = launches;
  return st;
}

int kda_fwd(const kda_problem* p, kda_dtype dtype, const void* q, const void* k, const void* v,
            const float* log_alpha, const void* beta, const float* w_text, const float* w_vis,
            const float* initial_state, void* o, float* final_state, void* workspace,
            size_t workspace_bytes_, void* stream) {
  g_last_launches = 0;
  kda::Dims d;
  int st = make_dims(p, dtype, &d);
  if (st) return st;
  if (d.reuse_records || d.qkv_f16) return KDA_ERR_INVALID_ARG;
  if ((st = check_ptrs({q, k, v, log_alpha, beta, w_text, w_vis, o}, {initial_state, final_state})))
    return st;
  if ((st = check_workspace(d, dtype, workspace, workspace_bytes_))) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws);
  const size_t act = align256(act_bytes(d, dtype));
  void* qc = ws + kStatusBytes;
  void* kc = ws + kStatusBytes + act;
  void* vc = ws + kStatusBytes + 2 * act;
  if ((st = cuda_status(cudaMemsetAsync(status, 0, sizeof(uint32_t), s)))) return st;
  int launches = 0;
  const bool tc = use_tc(d, dtype);
  if (d.N > 0) {
    st = cuda_status(kda::launch_shortconv(d, dtype, q, k, v, w_text, w_vis, qc, kc, vc, s, &launches, tc));
    if (st) return st;
  }
  st = run_scan(d, dtype, qc, kc, vc, log_alpha, beta, initial_state, o, final_state, workspace, s, &launches, tc);
  if (!st) g_last_launches = launches;
  return st;
}

size_t kda_bwd_workspace_bytes(const kda_problem* p, kda_dtype dtype) {
  kda::Dims d;
  if (make_dims(p, dtype, &d) || d.reuse_records || d.qkv_f16) return 0;
  return kda::bwd_workspace_bytes(d, dtype);
}

int kda_bwd(const kda_problem* p, kda_dtype dtype, const void* q, const void* k, const void* v,
            const float* log_alpha, const void* beta, const float* w_text, const float* w_vis,
            const float* initial_state, const void* d_o, const float* d_final_state, void* dq, void* dk, void* dv,
            float* d_log_alpha, void* d_beta, float* d_w_text, float* d_w_vis, float* d_initial_state,
            void* workspace, size_t workspace_bytes_, void* stream) {
  g_last_launches = 0;
  kda::Dims d;
  int st = make_dims(p, dtype, &d);
  if (st) return st;
  if (d.reuse_records || d.qkv_f16) return KDA_ERR_INVALID_ARG;
  if ((st = check_ptrs({q, k, v, log_alpha, beta, w_text, w_vis, d_o, dq, dk, dv, d_log_alpha, d_beta, d_w_text,
                        d_w_vis},
                       {initial_state, d_final_state, d_initial_state})))
    return st;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return KDA_ERR_WORKSPACE;
  if (workspace_bytes_ < kda::bwd_workspace_bytes(d, dtype)) return KDA_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((st = cuda_status(cudaMemsetAsync(workspace, 0, sizeof(uint32_t), s)))) return st;
  int launches = 0;
  st = cuda_status(kda::launch_bwd(d, dtype, q, k, v, log_alpha, beta, w_text, w_vis, initial_state, d_o,
                                   d_final_state, dq, dk, dv, d_log_alpha, d_beta, d_w_text, d_w_vis,
                                   d_initial_state, workspace, s, &launches));
  if (!st) g_last_launches = launches;
  return st;
}

int kda_read_status(void* workspace, void* stream) {
  if (!workspace) return KDA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t v = 0;
  if (cudaStreamSynchronize(s) != cudaSuccess) return KDA_ERR_CUDA;
  if (cudaMemcpy(&v, workspace, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return KDA_ERR_CUDA;
  if (cudaMemset(workspace, 0, sizeof(uint32_t)) != cudaSuccess) return KDA_ERR_CUDA;
  return (int)v;
}

const char* kda_status_str(int s) {
  switch (s) {
    case KDA_OK: return "ok";
    case KDA_ERR_INVALID_ARG: return "invalid argument";
    case KDA_ERR_UNSUPPORTED: return "unsupported problem size or option";
    case KDA_ERR_MISALIGNED: return "data pointer not 16-byte aligned";
    case KDA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case KDA_ERR_CUDA: return "CUDA runtime error";
    case KDA_ERR_TIMEOUT: return "device wait timed out";
    case KDA_ERR_DEVICE_ASSERT: return "device consistency check failed";
    case KDA_ERR_RANGE: return "gate decay within a chunk exceeds the bf16 tensor path's range";
    default: return "unknown status";
  }
}

int kda_last_launch_count(void) { return g_last_launches; }

}  // extern "C"
