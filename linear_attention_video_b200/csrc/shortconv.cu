// Modality-aware depthwise short convolution on q, k and v.
//
// Text tokens: causal 1D depthwise conv; visual tokens: depthwise 3D conv over
// the (T, H, W) latent grid, zero outside the grid, per modality (genai-atlas,
// "How it works"; paper.rainbus.top, section 核心方法).  fp32 accumulation,
// one rounding to the output type.
//
// Visual part (the bulk of the work, bound by the fp32 FMA pipe): a CTA owns
// 32 channels of one tensor and a tile of up to 4 rows x 64 columns of the
// grid, and slides through time.  Input planes (the tile plus a one-pixel halo)
// of three consecutive frames sit in shared memory as fp32, so each input
// element is read from global memory and converted once; the next plane's
// global loads are in flight while the current frame is computed.  A thread
// owns 2 channels (their 54 weights live in registers) and a run of up to 16
// pixels along a row, so every value it reads from shared memory feeds 3
// horizontal taps.
//
// Text part: a small kernel, one thread per (token, 8 channels).
#include <cuda_fp16.h>

#include "common.cuh"

namespace kda {
namespace {

constexpr int kVisTaps = 27;
constexpr int CG = 32;            // channels per CTA
constexpr int TH = 4;             // tile rows
constexpr int TWMAX = 64;         // tile columns
constexpr int PH = TH + 2, PW = TWMAX + 2;
constexpr int PLANE_FLOATS = PH * PW * CG;
constexpr int RUNMAX = TWMAX / 4;
constexpr int kThreads = 256;
constexpr int kPrefetch = (PH * PW * (CG / 8) + kThreads - 1) / kThreads;   // 16-byte chunks per thread

struct ConvArgs {
  const void* x[3];
  void* y[3];
  const float* w_text;  // [3][C][text_k]
  const float* w_vis;   // [3][C][27]
  int64_t N, L;
  int B, C, text_k;
  int T, Hg, Wg, pt;
  int n_wtiles, n_hbands;
};

// ---- type helpers ----------------------------------------------------------
template <typename T> struct Act;
template <> struct Act<__nv_bfloat16> {
  static __device__ __forceinline__ void widen8(uint4 u, float (&v)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
  static __device__ __forceinline__ uint32_t pack2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
  }
};
template <> struct Act<__half> {
  static __device__ __forceinline__ uint32_t pack2(float a, float b) {
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
  }
};
template <> struct Act<float> {};

// 8 consecutive channels of one token -> fp32
template <typename T> __device__ __forceinline__ void load8(const T* p, float (&v)[8]);
template <> __device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* p, float (&v)[8]) {
  Act<__nv_bfloat16>::widen8(__ldg(reinterpret_cast<const uint4*>(p)), v);
}
template <> __device__ __forceinline__ void load8<float>(const float* p, float (&v)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// store 2 consecutive channels
template <typename T> __device__ __forceinline__ void store2(T* p, float a, float b);
template <> __device__ __forceinline__ void store2<__nv_bfloat16>(__nv_bfloat16* p, float a, float b) {
  *reinterpret_cast<uint32_t*>(p) = Act<__nv_bfloat16>::pack2(a, b);
}
template <> __device__ __forceinline__ void store2<__half>(__half* p, float a, float b) {
  *reinterpret_cast<uint32_t*>(p) = Act<__half>::pack2(a, b);
}
template <> __device__ __forceinline__ void store2<float>(float* p, float a, float b) {
  *reinterpret_cast<float2*>(p) = make_float2(a, b);
}

// raw 16-byte chunk holding 8 channels (bf16: one uint4; fp32: two float4 -> handled separately)
template <typename T> struct Chunk { uint4 a; };
template <> struct Chunk<float> { float4 a, b; };

template <typename T> __device__ __forceinline__ void chunk_load(const T* p, Chunk<T>& c) {
  c.a = __ldg(reinterpret_cast<const uint4*>(p));
}
template <> __device__ __forceinline__ void chunk_load<float>(const float* p, Chunk<float>& c) {
  c.a = __ldg(reinterpret_cast<const float4*>(p));
  c.b = __ldg(reinterpret_cast<const float4*>(p) + 1);
}
template <typename T> __device__ __forceinline__ void chunk_zero(Chunk<T>& c) { c.a = make_uint4(0, 0, 0, 0); }
template <> __device__ __forceinline__ void chunk_zero<float>(Chunk<float>& c) {
  c.a = make_float4(0.f, 0.f, 0.f, 0.f);
  c.b = c.a;
}
template <typename T> __device__ __forceinline__ void chunk_store(float* dst, const Chunk<T>& c) {
  float v[8];
  Act<__nv_bfloat16>::widen8(c.a, v);
  reinterpret_cast<float4*>(dst)[0] = make_float4(v[0], v[1], v[2], v[3]);
  reinterpret_cast<float4*>(dst)[1] = make_float4(v[4], v[5], v[6], v[7]);
}
template <> __device__ __forceinline__ void chunk_store<float>(float* dst, const Chunk<float>& c) {
  reinterpret_cast<float4*>(dst)[0] = c.a;
  reinterpret_cast<float4*>(dst)[1] = c.b;
}

// ---- visual kernel -----------------------------------------------------------
// RUN: pixels per thread along a row (compile-time, so the FMA loop carries no
// predicates); a tile is 4 runs wide.  Columns past the grid edge read the zero
// padding of the plane and their outputs are not stored.
template <typename TIn, typename TOut, int RUN>
__global__ void __launch_bounds__(kThreads, 1) vis_conv_kernel(ConvArgs a) {
  extern __shared__ __align__(16) float planes[];   // [3][PH][PW][CG]
  const int tid = threadIdx.x;
  const int tile = blockIdx.x;
  const int wt = tile % a.n_wtiles, hb = tile / a.n_wtiles;
  const int cg0 = blockIdx.y * CG;
  const int tensor = blockIdx.z % 3, b = blockIdx.z / 3;
  const int C = a.C;
  const int tw0 = wt * (4 * RUN), th0 = hb * TH;
  const int TW = min(4 * RUN, a.Wg - tw0), THh = min(TH, a.Hg - th0);
  const int64_t HW = (int64_t)a.Hg * a.Wg;
  const TIn* x = static_cast<const TIn*>(a.x[tensor]) + ((int64_t)b * a.N + a.L) * C + cg0;
  TOut* y = static_cast<TOut*>(a.y[tensor]) + ((int64_t)b * a.N + a.L) * C + cg0;

  // thread roles
  const int cp = tid & 15;              // channel pair
  const int wk = tid >> 4;              // worker 0..15: row wk&3, run wk>>2
  const int row = wk & 3, run = wk >> 2;
  const int w0 = run * RUN;
  const int nrun = max(0, min(RUN, TW - w0));
  const bool active = row < THh && nrun > 0;

  // weights of channels cg0+2cp, +1
  float wv0[kVisTaps], wv1[kVisTaps];
  {
    const float* wbase = a.w_vis + ((int64_t)tensor * C + cg0 + 2 * cp) * kVisTaps;
#pragma unroll
    for (int i = 0; i < kVisTaps; ++i) {
      wv0[i] = wbase[i];
      wv1[i] = wbase[kVisTaps + i];
    }
  }

  // plane loader: chunk index e -> (prow, pcol, channel block of 8)
  const int PWr = 4 * RUN + 2;                       // plane columns read by the runs (incl. halo)
  const int n_chunks = PH * PWr * (CG / 8);
  auto plane_fetch = [&](int f, Chunk<TIn> (&buf)[kPrefetch]) {
#pragma unroll
    for (int i = 0; i < kPrefetch; ++i) {
      const int e = tid + i * kThreads;
      chunk_zero<TIn>(buf[i]);
      if (e < n_chunks && f >= 0 && f < a.T) {
        const int cb = e & 3, pix = e >> 2;
        const int pr = pix / PWr, pc = pix - pr * PWr;
        const int hh = th0 + pr - 1, ww = tw0 + pc - 1;
        if (hh >= 0 && hh < a.Hg && ww >= 0 && ww < a.Wg)
          chunk_load<TIn>(x + ((int64_t)f * HW + (int64_t)hh * a.Wg + ww) * C + cb * 8, buf[i]);
      }
    }
  };
  auto plane_store = [&](int f, const Chunk<TIn> (&buf)[kPrefetch]) {
    float* pl = planes + (((f % 3) + 3) % 3) * PLANE_FLOATS;
#pragma unroll
    for (int i = 0; i < kPrefetch; ++i) {
      const int e = tid + i * kThreads;
      if (e < n_chunks) {
        const int cb = e & 3, pix = e >> 2;
        const int pr = pix / PWr, pc = pix - pr * PWr;
        chunk_store<TIn>(pl + (pr * PW + pc) * CG + cb * 8, buf[i]);
      }
    }
  };

  // Frame t reads planes t-pt .. t+2-pt.  Three plane slots in shared memory
  // (slot = frame mod 3) plus one plane in flight in registers.
  Chunk<TIn> buf[kPrefetch];
  for (int f = -a.pt; f <= 2 - a.pt; ++f) {
    plane_fetch(f, buf);
    plane_store(f, buf);
  }
  __syncthreads();

  for (int t = 0; t < a.T; ++t) {
    const int f_next = t + 3 - a.pt;   // first plane frame t+1 needs that is not resident
    plane_fetch(f_next, buf);          // global loads overlap the compute of frame t
    if (active) {
      float acc0[RUN], acc1[RUN];
#pragma unroll
      for (int i = 0; i < RUN; ++i) { acc0[i] = 0.f; acc1[i] = 0.f; }
#pragma unroll
      for (int ta = 0; ta < 3; ++ta) {
        const int f = t + ta - a.pt;
        if (f < 0 || f >= a.T) continue;
        const float* pl = planes + (f % 3) * PLANE_FLOATS;
#pragma unroll
        for (int tb = 0; tb < 3; ++tb) {
          const float2* src = reinterpret_cast<const float2*>(pl + ((row + tb) * PW + w0) * CG + 2 * cp);
          float2 in[RUN + 2];
#pragma unroll
          for (int i = 0; i < RUN + 2; ++i) in[i] = src[i * (CG / 2)];
#pragma unroll
          for (int te = 0; te < 3; ++te) {
            const float c0 = wv0[(ta * 3 + tb) * 3 + te], c1 = wv1[(ta * 3 + tb) * 3 + te];
#pragma unroll
            for (int i = 0; i < RUN; ++i) {
              acc0[i] = fmaf(c0, in[i + te].x, acc0[i]);
              acc1[i] = fmaf(c1, in[i + te].y, acc1[i]);
            }
          }
        }
      }
      TOut* yo = y + ((int64_t)t * HW + (int64_t)(th0 + row) * a.Wg + tw0 + w0) * C + 2 * cp;
#pragma unroll
      for (int i = 0; i < RUN; ++i)
        if (i < nrun) store2<TOut>(yo + (int64_t)i * C, acc0[i], acc1[i]);
    }
    __syncthreads();                   // every thread is done with the slot of frame t-pt
    plane_store(f_next, buf);
    __syncthreads();
  }
}

// ---- text kernel -------------------------------------------------------------
template <typename TIn, typename TOut>
__global__ void __launch_bounds__(256) text_conv_kernel(ConvArgs a) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;   // over B * L * (C/8)
  const int tensor = blockIdx.y;
  const int C = a.C, C8 = C / 8;
  const int64_t total = (int64_t)a.B * a.L * C8;
  if (idx >= total) return;
  const int c0 = (int)(idx % C8) * 8;
  const int64_t bt = idx / C8;
  const int64_t b = bt / a.L, n = bt - b * a.L;
  const TIn* x = static_cast<const TIn*>(a.x[tensor]) + b * a.N * C;
  TOut* y = static_cast<TOut*>(a.y[tensor]) + b * a.N * C;
  const float* w = a.w_text + ((int64_t)tensor * C + c0) * a.text_k;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (int j = 0; j < a.text_k; ++j) {
    const int64_t src = n - (a.text_k - 1) + j;
    if (src < 0) continue;
    float v[8];
    load8<TIn>(x + src * C + c0, v);
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = fmaf(w[e * a.text_k + j], v[e], acc[e]);
  }
#pragma unroll
  for (int e = 0; e < 8; e += 2) store2<TOut>(y + n * C + c0 + e, acc[e], acc[e + 1]);
}

template <typename TIn, typename TOut, int RUN>
cudaError_t launch_vis(const ConvArgs& a0, cudaStream_t s) {
  ConvArgs a = a0;
  a.n_wtiles = (a.Wg + 4 * RUN - 1) / (4 * RUN);
  const size_t smem = 3 * PLANE_FLOATS * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(vis_conv_kernel<TIn, TOut, RUN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)(a.n_wtiles * a.n_hbands), (unsigned)(a.C / CG), (unsigned)(3 * a.B));
  vis_conv_kernel<TIn, TOut, RUN><<<grid, kThreads, smem, s>>>(a);
  return cudaGetLastError();
}

template <typename TIn, typename TOut>
cudaError_t launch_t(const ConvArgs& a, cudaStream_t s) {
  if (a.L > 0) {
    const int64_t total = (int64_t)a.B * a.L * (a.C / 8);
    text_conv_kernel<TIn, TOut><<<dim3((unsigned)((total + 255) / 256), 3), 256, 0, s>>>(a);
  }
  if (a.T > 0) {
    // widest run whose tiles cover the row with the least padding
    if (a.Wg % 52 == 0 || (a.Wg <= 52 && a.Wg > 48)) return launch_vis<TIn, TOut, 13>(a, s);
    if (a.Wg % 64 == 0 || a.Wg > 52) return launch_vis<TIn, TOut, 16>(a, s);
    return launch_vis<TIn, TOut, 8>(a, s);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_shortconv(const Dims& d, kda_dtype dt, const void* q, const void* k, const void* v,
                             const float* w_text, const float* w_vis, void* qo, void* ko, void* vo,
                             cudaStream_t s, int* launches, bool out_f16) {
  ConvArgs a;
  a.x[0] = q; a.x[1] = k; a.x[2] = v;
  a.y[0] = qo; a.y[1] = ko; a.y[2] = vo;
  a.w_text = w_text; a.w_vis = w_vis;
  a.N = d.N; a.L = d.L; a.B = d.B;
  a.C = d.H * d.dk;
  a.text_k = d.text_k;
  a.T = d.T; a.Hg = d.Hg; a.Wg = d.Wg; a.pt = d.pt;
  a.n_wtiles = d.T > 0 ? (d.Wg + TWMAX - 1) / TWMAX : 0;
  a.n_hbands = d.T > 0 ? (d.Hg + TH - 1) / TH : 0;
  if ((int64_t)d.B * d.N == 0) return cudaSuccess;
  cudaError_t e;
  if (dt == KDA_DT_BF16 && out_f16) e = launch_t<__nv_bfloat16, __half>(a, s);
  else if (dt == KDA_DT_BF16) e = launch_t<__nv_bfloat16, __nv_bfloat16>(a, s);
  else e = launch_t<float, float>(a, s);
  if (e == cudaSuccess && launches) *launches += (a.L > 0) + (a.T > 0);
  return e;
}

}  // namespace kda
