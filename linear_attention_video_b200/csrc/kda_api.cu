// C-ABI layer: argument validation, workspace layout, dispatch to the kernels.
// The operations and layouts are documented in include/kda.h.
#include <string.h>

#include <algorithm>
#include <vector>

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
  // the tensor-core scan (bf16, d = 128) works on 64-token sub-chunks composed into 128-token blocks
  if (dt == KDA_DT_BF16 && kda::chunk_tc_supported(*d) && d->chunk != 64) return KDA_ERR_UNSUPPORTED;
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

// ---- kda_fwd on host-resident tensors -------------------------------------------------
// The token stream of each batch item is cut into segments of seg_frames visual frames (the
// text prefix goes with the first).  Per segment: its inputs are copied in on the copy-in
// stream, its conv and scan run on the caller's stream (the scan entering with the state the
// previous segment left), and its o is copied out on the copy-out stream; events order the
// three, so copies of neighbouring segments overlap the kernels.  The conv of a segment reads
// the neighbouring frames its taps reach (pt before, 2 - pt after): its view is that frame range,
// and the outputs it computes for the halo frames (with zeros beyond the view) are discarded:
// the earlier segment has already used its own, and the next one recomputes them first.
struct HostLayout {
  size_t act, la, beta, state, rec, total;
};

kda::Dims segment_dims(const kda::Dims& d, int64_t n_tokens) {   // a 1-item, text-only view of n tokens
  kda::Dims s = d;
  s.B = 1;
  s.N = n_tokens;
  s.L = n_tokens;
  s.T = s.Hg = s.Wg = 0;
  return s;
}

int64_t max_segment_tokens(const kda::Dims& d, int seg_frames) {
  return d.L + (int64_t)std::min(seg_frames, d.T) * d.Hg * d.Wg;
}

// status | q, k, v, log alpha, beta, o staged on the device | q', k', v' | two per-item states | scan records
HostLayout host_layout(const kda::Dims& d, kda_dtype dt, int seg_frames) {
  HostLayout l;
  l.act = align256(act_bytes(d, dt));
  l.la = align256((size_t)d.B * d.N * d.H * d.dk * sizeof(float));
  l.beta = align256((size_t)d.B * d.N * d.H * elem_size(dt));
  l.state = align256((size_t)d.H * d.dk * d.dv * sizeof(float));
  l.rec = use_tc(d, dt) ? align256(kda::chunk_tc_workspace_bytes(segment_dims(d, max_segment_tokens(d, seg_frames))))
                        : 0;
  l.total = kStatusBytes + 7 * l.act + l.la + l.beta + 2 * l.state + l.rec;
  return l;
}

}  // namespace

namespace kda {
// Validation shared with the allocation-free entry point (noalloc.cu).
int validate_problem(const kda_problem* p, kda_dtype dt, Dims* d) { return make_dims(p, dt, d); }
int validate_scan_pointers(const void* q, const void* k, const void* v, const void* la, const void* beta, const void* o,
                           const void* s0, const void* sn) {
  return check_ptrs({q, k, v, la, beta, o}, {s0, sn});
}
void set_last_launch_count(int launches) { g_last_launches = launches; }
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

size_t kda_fwd_host_workspace_bytes(const kda_problem* p, kda_dtype dtype, int32_t seg_frames) {
  kda::Dims d;
  if (make_dims(p, dtype, &d) != KDA_OK || d.reuse_records || d.qkv_f16 || seg_frames < 1) return 0;
  return host_layout(d, dtype, seg_frames).total;
}

int kda_fwd_host(const kda_problem* p, kda_dtype dtype, const void* q, const void* k, const void* v,
                 const float* log_alpha, const void* beta, const float* w_text, const float* w_vis,
                 const float* initial_state, void* o, float* final_state, int32_t seg_frames, void* workspace,
                 size_t workspace_bytes_, void* stream, void* copy_in_stream, void* copy_out_stream) {
  g_last_launches = 0;
  kda::Dims d;
  int st = make_dims(p, dtype, &d);
  if (st) return st;
  if (d.reuse_records || d.qkv_f16 || seg_frames < 1) return KDA_ERR_INVALID_ARG;
  if ((st = check_ptrs({q, k, v, log_alpha, beta, w_text, w_vis, o}, {initial_state, final_state}))) return st;
  const HostLayout l = host_layout(d, dtype, seg_frames);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes_ < l.total)
    return KDA_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaStream_t cin = static_cast<cudaStream_t>(copy_in_stream), cout = static_cast<cudaStream_t>(copy_out_stream);
  char* ws = static_cast<char*>(workspace);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws);
  char* base = ws + kStatusBytes;
  char* dq = base;                  // staged inputs and output, layouts as in kda_fwd
  char* dk = dq + l.act;
  char* dv = dk + l.act;
  char* dout = dv + l.act;
  char* qc = dout + l.act;          // conv outputs (fp16 on the tensor-core path)
  char* kc = qc + l.act;
  char* vc = kc + l.act;
  float* dla = reinterpret_cast<float*>(vc + l.act);
  char* dbeta = reinterpret_cast<char*>(dla) + l.la;
  float* state[2] = {reinterpret_cast<float*>(dbeta + l.beta), reinterpret_cast<float*>(dbeta + l.beta + l.state)};
  void* rec = dbeta + l.beta + 2 * l.state;
  const bool tc = use_tc(d, dtype);
  const size_t es = elem_size(dtype), row = (size_t)d.H * d.dk;   // one token of q, k, v, o: row elements
  const int64_t HW = (int64_t)d.Hg * d.Wg;
  const int before = d.pt, after = 2 - d.pt;                      // frames the conv taps reach
  const int nseg_item = d.T > 0 ? (d.T + seg_frames - 1) / seg_frames : 1;
  const int nseg = d.B * nseg_item;
  if ((st = cuda_status(cudaMemsetAsync(status, 0, sizeof(uint32_t), s)))) return st;

  std::vector<cudaEvent_t> ev(2 * nseg + 2, nullptr);
  auto cleanup = [&]() {
    for (cudaEvent_t e : ev)
      if (e) cudaEventDestroy(e);   // released once the work they mark completes
  };
  for (cudaEvent_t& e : ev)
    if ((st = cuda_status(cudaEventCreateWithFlags(&e, cudaEventDisableTiming)))) { cleanup(); return st; }
  cudaEvent_t* ev_in = ev.data();
  cudaEvent_t* ev_comp = ev.data() + nseg;
  cudaEvent_t ev_start = ev[2 * nseg], ev_done = ev[2 * nseg + 1];
  int launches = 0;
  auto fail = [&](cudaError_t e) { cleanup(); return cuda_status(e); };
  cudaError_t e;
  // the copies wait for the caller's stream: earlier work there may still read the workspace
  if ((e = cudaEventRecord(ev_start, s)) != cudaSuccess || (e = cudaStreamWaitEvent(cin, ev_start, 0)) != cudaSuccess)
    return fail(e);
  for (int b = 0; b < d.B; ++b) {
    const int64_t item = (int64_t)b * d.N;   // first token of the item
    int64_t copied = 0;                      // q, k, v tokens of the item already copied in
    const size_t sbytes = (size_t)d.H * d.dk * d.dv * sizeof(float);
    const float* S_in = initial_state ? initial_state + (size_t)b * d.H * d.dk * d.dv : nullptr;
    if (d.N == 0) {   // nothing to scan: the state passes through
      float* SN = final_state ? final_state + (size_t)b * d.H * d.dk * d.dv : nullptr;
      if (SN && (e = S_in ? cudaMemcpyAsync(SN, S_in, sbytes, cudaMemcpyDeviceToDevice, s)
                          : cudaMemsetAsync(SN, 0, sbytes, s)) != cudaSuccess)
        return fail(e);
      continue;
    }
    for (int sg = 0; sg < nseg_item; ++sg) {
      const int id = b * nseg_item + sg;
      const int f0 = sg * seg_frames, f1 = std::min(d.T, f0 + seg_frames);
      const int64_t s_lo = f0 == 0 ? 0 : d.L + f0 * HW, s_hi = d.L + f1 * HW;   // this segment's tokens
      const int fv0 = std::max(0, f0 - before), fv1 = std::min(d.T, f1 + after);
      const int64_t v_lo = f0 == 0 ? 0 : d.L + fv0 * HW, v_hi = d.L + fv1 * HW;   // tokens the conv reads
      // copy in: q, k, v up to the conv's last frame, log alpha and beta of the segment
      if (v_hi > copied) {
        const size_t off = (size_t)(item + copied) * row * es, n = (size_t)(v_hi - copied) * row * es;
        for (int t = 0; t < 3; ++t) {
          const void* src = t == 0 ? q : (t == 1 ? k : v);
          char* dst = t == 0 ? dq : (t == 1 ? dk : dv);
          if ((e = cudaMemcpyAsync(dst + off, static_cast<const char*>(src) + off, n, cudaMemcpyHostToDevice, cin)) !=
              cudaSuccess)
            return fail(e);
        }
        copied = v_hi;
      }
      {
        const size_t t0 = (size_t)(item + s_lo), nt = (size_t)(s_hi - s_lo);
        if ((e = cudaMemcpyAsync(dla + t0 * row, log_alpha + t0 * row, nt * row * sizeof(float), cudaMemcpyHostToDevice,
                                 cin)) != cudaSuccess ||
            (e = cudaMemcpyAsync(dbeta + t0 * d.H * es, static_cast<const char*>(beta) + t0 * d.H * es, nt * d.H * es,
                                 cudaMemcpyHostToDevice, cin)) != cudaSuccess ||
            (e = cudaEventRecord(ev_in[id], cin)) != cudaSuccess)
          return fail(e);
      }
      // compute: the conv over the view, then the scan over the segment's tokens
      if ((e = cudaStreamWaitEvent(s, ev_in[id], 0)) != cudaSuccess) return fail(e);
      {
        kda::Dims dvw = d;
        dvw.B = 1;
        dvw.L = f0 == 0 ? d.L : 0;
        dvw.T = fv1 - fv0;
        dvw.N = dvw.L + (int64_t)dvw.T * HW;
        const size_t off = (size_t)(item + v_lo) * row * es;
        if ((e = kda::launch_shortconv(dvw, dtype, dq + off, dk + off, dv + off, w_text, w_vis, qc + off, kc + off,
                                       vc + off, s, &launches, tc)) != cudaSuccess)
          return fail(e);
      }
      {
        const kda::Dims dsg = segment_dims(d, s_hi - s_lo);
        const size_t t0 = (size_t)(item + s_lo), off = t0 * row * es;
        const bool last = sg == nseg_item - 1;
        float* S_out = last ? (final_state ? final_state + (size_t)b * d.H * d.dk * d.dv : nullptr) : state[sg & 1];
        e = tc ? kda::launch_chunk_tc(dsg, true, qc + off, kc + off, vc + off, dla + t0 * row, dbeta + t0 * d.H * es,
                                      S_in, dout + off, S_out, rec, status, s, &launches)
               : kda::launch_chunk_simt(dsg, dtype, qc + off, kc + off, vc + off, dla + t0 * row, dbeta + t0 * d.H * es,
                                        S_in, dout + off, S_out, status, s, &launches);
        if (e != cudaSuccess || (e = cudaEventRecord(ev_comp[id], s)) != cudaSuccess) return fail(e);
        S_in = S_out;
      }
      // copy out
      {
        const size_t off = (size_t)(item + s_lo) * row * es, n = (size_t)(s_hi - s_lo) * row * es;
        if ((e = cudaStreamWaitEvent(cout, ev_comp[id], 0)) != cudaSuccess ||
            (e = cudaMemcpyAsync(static_cast<char*>(o) + off, dout + off, n, cudaMemcpyDeviceToHost, cout)) !=
                cudaSuccess)
          return fail(e);
      }
    }
  }
  // the caller's stream covers everything the call enqueued
  if ((e = cudaEventRecord(ev_done, cout)) != cudaSuccess || (e = cudaStreamWaitEvent(s, ev_done, 0)) != cudaSuccess)
    return fail(e);
  cleanup();
  g_last_launches = launches;
  return KDA_OK;
}

int kda_selftest_wait_timeout(const kda_problem* p, kda_dtype dtype, const void* q, const void* k, const void* v,
                              const float* log_alpha, const void* beta, void* o, void* workspace,
                              size_t workspace_bytes_, int32_t stage, uint32_t wait_us, void* stream) {
  g_last_launches = 0;
  kda::Dims d;
  int st = make_dims(p, dtype, &d);
  if (st) return st;
  if (!use_tc(d, dtype) || d.reuse_records || d.N == 0) return KDA_ERR_UNSUPPORTED;
  if ((stage != 1 && stage != 2) || wait_us < 1) return KDA_ERR_INVALID_ARG;
  if ((st = check_ptrs({q, k, v, log_alpha, beta, o}, {}))) return st;
  if ((st = check_workspace(d, dtype, workspace, workspace_bytes_))) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t* status = static_cast<uint32_t*>(workspace);
  if ((st = cuda_status(cudaMemsetAsync(status, 0, sizeof(uint32_t), s)))) return st;
  int launches = 0;
  void* rec = static_cast<char*>(workspace) + tc_records_offset(d, dtype);
  st = cuda_status(kda::launch_chunk_tc(d, d.qkv_f16, q, k, v, log_alpha, beta, nullptr, o, nullptr, rec, status, s,
                                        &launches, stage, (uint64_t)wait_us * 1000ull));
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
    case KDA_ERR_RANGE: return "gate decay within a chunk exceeds the backward pass's range";
    default: return "unknown status";
  }
}

int kda_last_launch_count(void) { return g_last_launches; }

}  // extern "C"
