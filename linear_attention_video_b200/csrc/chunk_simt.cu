// Chunked KDA scan in fp32 on the CUDA cores (the fp32 path; exact to ~1e-6).
//
// Recurrence (paper.rainbus.top, section 方法步骤详情 step (5)):
//   S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,  o_t = S_t^T q_t.
// Chunked form, per chunk of n <= CH tokens entering with state S, with
// g_r = sum_{i<=r} log alpha_i (within the chunk, per key channel):
//   A[r,i] = beta_r sum_c k_rc k_ic e^{g_rc - g_ic}  (i < r)
//   P[r,i] = sum_c q_rc k_ic e^{g_rc - g_ic}         (i <= r)
//   [W | U~] = (I + A)^{-1} Diag(beta) [K*e^g | V]
//   U = U~ - W S;   O = (Q*e^g) S + P U;   S <- Diag(e^{g_last}) S + (K*e^{g_last-g})^T U
// Padding rows of the last chunk carry k = q = v = 0, beta = 0, log alpha = 0,
// which leaves all of the above unchanged.
//
// One CTA per (batch item, head, slice of DVS value columns): columns of S
// evolve independently.  e^{g_r - g_i} is formed as e^{g_r} * e^{-g_i} when every
// channel's decay over the chunk is at most 80 nats (no overflow); otherwise
// the chunk takes the exact pairwise-exponential branch.
#include "common.cuh"

namespace kda {
namespace {

constexpr int kThreads = 256;
constexpr int DVS = 32;            // value columns per CTA
constexpr float kSafeDecay = 80.f;

template <int DK, int CH>
struct SimtSmem {
  static constexpr int LD = DK + 1;   // padded row stride of the [CH][DK] buffers
  static constexpr size_t floats = 4 * CH * LD + 2 * CH * CH + CH * DVS + DK * DVS + CH + DK + 4;
  static constexpr size_t bytes = floats * sizeof(float);
};

template <typename T, int DK, int CH>
__global__ void __launch_bounds__(kThreads) chunk_simt_kernel(
    const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
    const float* __restrict__ la, const T* __restrict__ beta,
    const float* __restrict__ S0, T* __restrict__ o, float* __restrict__ SN,
    int64_t N, int H, int dv, uint32_t* status) {
  using L = SimtSmem<DK, CH>;
  constexpr int LD = L::LD;
  extern __shared__ float smem[];
  float* B0 = smem;                 // [CH][LD]
  float* B1 = B0 + CH * LD;
  float* B2 = B1 + CH * LD;
  float* B3 = B2 + CH * LD;
  float* Am = B3 + CH * LD;         // [CH][CH]
  float* Pm = Am + CH * CH;         // [CH][CH]
  float* Vs = Pm + CH * CH;         // [CH][DVS]   V -> U~ -> U
  float* Ss = Vs + CH * DVS;        // [DK][DVS]
  float* bs = Ss + DK * DVS;        // [CH]
  float* gl = bs + CH;              // [DK]   g_last

  const int tid = threadIdx.x;
  const int j0 = blockIdx.x * DVS;
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const int64_t tok_stride_k = (int64_t)H * DK;   // stride between tokens in q, k, la
  const int64_t tok_stride_v = (int64_t)H * dv;   // stride between tokens in v, o
  const T* qb = q + (int64_t)b * N * tok_stride_k + (int64_t)h * DK;
  const T* kb = k + (int64_t)b * N * tok_stride_k + (int64_t)h * DK;
  const float* lab = la + (int64_t)b * N * tok_stride_k + (int64_t)h * DK;
  const T* vb = v + (int64_t)b * N * tok_stride_v + (int64_t)h * dv + j0;
  T* ob = o + (int64_t)b * N * tok_stride_v + (int64_t)h * dv + j0;
  const T* bb = beta + (int64_t)b * N * H + h;

  // state slice S[c][j], j in [j0, j0+DVS)
  for (int i = tid; i < DK * DVS; i += kThreads) {
    const int c = i / DVS, j = i % DVS;
    Ss[i] = S0 ? S0[(((int64_t)b * H + h) * DK + c) * dv + j0 + j] : 0.f;
  }

  for (int64_t n0 = 0; n0 < N; n0 += CH) {
    const int n = (int)min((int64_t)CH, N - n0);
    __syncthreads();
    // ---- load K, Q (raw), V slice, beta; prefix sums of log alpha ----
    for (int i = tid; i < CH * DK; i += kThreads) {
      const int r = i / DK, c = i % DK;
      float kv = 0.f, qv = 0.f;
      if (r < n) {
        kv = to_f32(kb[(n0 + r) * tok_stride_k + c]);
        qv = to_f32(qb[(n0 + r) * tok_stride_k + c]);
      }
      B0[r * LD + c] = kv;
      B1[r * LD + c] = qv;
    }
    for (int i = tid; i < CH * DVS; i += kThreads) {
      const int r = i / DVS, j = i % DVS;
      Vs[i] = r < n ? to_f32(vb[(n0 + r) * tok_stride_v + j]) : 0.f;
    }
    for (int r = tid; r < CH; r += kThreads) bs[r] = r < n ? to_f32(bb[(n0 + r) * H]) : 0.f;
    if (tid < DK) {
      float g = 0.f;
      for (int r = 0; r < CH; ++r) {
        if (r < n) g += lab[(n0 + r) * tok_stride_k + tid];
        B2[r * LD + tid] = g;
      }
      gl[tid] = g;
    }
    __syncthreads();
    const bool unsafe = __syncthreads_or(tid < DK && -gl[tid] > kSafeDecay);

    float* Wb;  // K*e^g, becomes W
    float* Kt;  // K*e^{g_last - g}
    float* Qg;  // Q*e^g
    if (!unsafe) {
      // B3 = K e^{-g}, B2 = K e^{g}, B1 = Q e^{g}
      for (int i = tid; i < CH * DK; i += kThreads) {
        const int r = i / DK, c = i % DK;
        const float g = B2[r * LD + c], kv = B0[r * LD + c];
        const float eg = __expf(g), emg = __expf(-g);
        B3[r * LD + c] = kv * emg;
        B2[r * LD + c] = kv * eg;
        B1[r * LD + c] *= eg;
      }
      __syncthreads();
      // A[r,i] = beta_r <K e^g_r, K e^-g_i>, P[r,i] = <Q e^g_r, K e^-g_i>
      for (int e = tid; e < CH * CH; e += kThreads) {
        const int r = e / CH, i = e % CH;
        float a = 0.f, p = 0.f;
        if (i <= r) {
          const float* kr = B2 + r * LD;
          const float* qr = B1 + r * LD;
          const float* ki = B3 + i * LD;
#pragma unroll 8
          for (int c = 0; c < DK; ++c) {
            a += kr[c] * ki[c];
            p += qr[c] * ki[c];
          }
        }
        Am[e] = i < r ? bs[r] * a : 0.f;
        Pm[e] = i <= r ? p : 0.f;
      }
      __syncthreads();
      // K~ = (K e^{-g}) e^{g_last} into B0
      for (int i = tid; i < CH * DK; i += kThreads) {
        const int r = i / DK, c = i % DK;
        B0[r * LD + c] = B3[r * LD + c] * __expf(gl[c]);
      }
      Wb = B2; Kt = B0; Qg = B1;
    } else {
      // exact pairwise exponentials
      for (int e = tid; e < CH * CH; e += kThreads) {
        const int r = e / CH, i = e % CH;
        float a = 0.f, p = 0.f;
        if (i <= r) {
          for (int c = 0; c < DK; ++c) {
            const float w = expf(B2[r * LD + c] - B2[i * LD + c]);
            a += B0[r * LD + c] * B0[i * LD + c] * w;
            p += B1[r * LD + c] * B0[i * LD + c] * w;
          }
        }
        Am[e] = i < r ? bs[r] * a : 0.f;
        Pm[e] = i <= r ? p : 0.f;
      }
      __syncthreads();
      for (int i = tid; i < CH * DK; i += kThreads) {
        const int r = i / DK, c = i % DK;
        const float g = B2[r * LD + c], kv = B0[r * LD + c];
        const float eg = expf(g);
        B3[r * LD + c] = kv * eg;
        B0[r * LD + c] = kv * expf(gl[c] - g);
        B1[r * LD + c] *= eg;
      }
      Wb = B3; Kt = B0; Qg = B1;
    }
    __syncthreads();

    // ---- [W | U~] = (I + A)^{-1} Diag(beta) [K e^g | V]: one column per thread ----
    for (int col = tid; col < DK + DVS; col += kThreads) {
      float* base = col < DK ? Wb + col : Vs + (col - DK);
      const int ld = col < DK ? LD : DVS;
      for (int r = 0; r < CH; ++r) {
        float y = bs[r] * base[r * ld];
        const float* ar = Am + r * CH;
        for (int jj = 0; jj < r; ++jj) y -= ar[jj] * base[jj * ld];
        base[r * ld] = y;
      }
    }
    __syncthreads();

    // ---- U = U~ - W S (in place in Vs) ----
    {
      const int j = tid % DVS;
      for (int r = tid / DVS; r < CH; r += kThreads / DVS) {
        float acc = 0.f;
        const float* wr = Wb + r * LD;
#pragma unroll 8
        for (int c = 0; c < DK; ++c) acc += wr[c] * Ss[c * DVS + j];
        Vs[r * DVS + j] -= acc;
      }
    }
    __syncthreads();

    // ---- O = (Q e^g) S + P U ----
    {
      const int j = tid % DVS;
      for (int r = tid / DVS; r < n; r += kThreads / DVS) {
        float acc = 0.f;
        const float* qr = Qg + r * LD;
#pragma unroll 8
        for (int c = 0; c < DK; ++c) acc += qr[c] * Ss[c * DVS + j];
        const float* pr = Pm + r * CH;
        for (int i = 0; i <= r; ++i) acc += pr[i] * Vs[i * DVS + j];
        ob[(n0 + r) * tok_stride_v + j] = from_f32<T>(acc);
      }
    }
    __syncthreads();

    // ---- S <- Diag(e^{g_last}) S + K~^T U ----
    {
      const int j = tid % DVS;
      for (int c = tid / DVS; c < DK; c += kThreads / DVS) {
        float acc = Ss[c * DVS + j] * __expf(gl[c]);
        for (int r = 0; r < CH; ++r) acc += Kt[r * LD + c] * Vs[r * DVS + j];
        Ss[c * DVS + j] = acc;
      }
    }
  }
  __syncthreads();
  if (SN)
    for (int i = tid; i < DK * DVS; i += kThreads) {
      const int c = i / DVS, j = i % DVS;
      SN[(((int64_t)b * H + h) * DK + c) * dv + j0 + j] = Ss[i];
    }
}

template <typename T, int DK, int CH>
cudaError_t launch_t(const Dims& d, const void* q, const void* k, const void* v, const float* la,
                     const void* beta, const float* S0, void* o, float* SN, uint32_t* status,
                     cudaStream_t s) {
  const size_t smem = SimtSmem<DK, CH>::bytes;
  auto kern = chunk_simt_kernel<T, DK, CH>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(d.dv / DVS, d.H, d.B);
  kern<<<grid, kThreads, smem, s>>>(static_cast<const T*>(q), static_cast<const T*>(k),
                                    static_cast<const T*>(v), la, static_cast<const T*>(beta), S0,
                                    static_cast<T*>(o), SN, d.N, d.H, d.dv, status);
  return cudaGetLastError();
}

template <typename T>
cudaError_t dispatch(const Dims& d, const void* q, const void* k, const void* v, const float* la,
                     const void* beta, const float* S0, void* o, float* SN, uint32_t* status,
                     cudaStream_t s) {
#define KDA_SIMT_CASE(DK_, CH_) \
  if (d.dk == DK_ && d.chunk == CH_) return launch_t<T, DK_, CH_>(d, q, k, v, la, beta, S0, o, SN, status, s);
  KDA_SIMT_CASE(64, 16) KDA_SIMT_CASE(64, 32) KDA_SIMT_CASE(64, 64)
  KDA_SIMT_CASE(128, 16) KDA_SIMT_CASE(128, 32) KDA_SIMT_CASE(128, 64)
#undef KDA_SIMT_CASE
  return cudaErrorInvalidValue;
}

}  // namespace

size_t chunk_simt_smem_bytes(int dk, int chunk) {
  if (dk == 64) return chunk == 16 ? SimtSmem<64, 16>::bytes : chunk == 32 ? SimtSmem<64, 32>::bytes : SimtSmem<64, 64>::bytes;
  return chunk == 16 ? SimtSmem<128, 16>::bytes : chunk == 32 ? SimtSmem<128, 32>::bytes : SimtSmem<128, 64>::bytes;
}

cudaError_t launch_chunk_simt(const Dims& d, kda_dtype dt, const void* q, const void* k, const void* v,
                              const float* log_alpha, const void* beta, const float* S0, void* o,
                              float* SN, uint32_t* status, cudaStream_t s, int* launches) {
  if (d.N == 0) return cudaSuccess;  // nothing to scan; final state handled by the caller
  cudaError_t e = dt == KDA_DT_BF16
                      ? dispatch<__nv_bfloat16>(d, q, k, v, log_alpha, beta, S0, o, SN, status, s)
                      : dispatch<float>(d, q, k, v, log_alpha, beta, S0, o, SN, status, s);
  if (e == cudaSuccess && launches) ++*launches;
  return e;
}

}  // namespace kda
