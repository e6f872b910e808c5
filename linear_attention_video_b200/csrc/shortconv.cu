// Modality-aware depthwise short convolution on q, k and v.
//
// Text tokens: causal 1D depthwise conv; visual tokens: depthwise 3D conv over
// the (T, H, W) latent grid, zero outside the grid, per modality (genai-atlas,
// "How it works"; paper.rainbus.top, section 核心方法).  fp32 accumulation,
// one rounding to the output type.
//
// Layout: x, y are [B, N, C] with C = H*d channels contiguous per token.  A
// block owns 256 consecutive channels of one tensor (q, k or v) and walks a
// range of tokens; a warp covers the 256 channels of one token (32 lanes x 8
// channels = 512 B of bf16), so every tap is one coalesced 16-byte load per
// lane.  The block's weights are staged transposed in shared memory
// ([tap][channel]) so each lane reads its 8 weights of a tap as two 16-byte
// shared loads.
#include <cuda_fp16.h>

#include "common.cuh"

namespace kda {
namespace {

constexpr int kChanPerBlock = 256;
constexpr int kTokPerBlock = 64;
constexpr int kMaxTextK = 8;
constexpr int kVisTaps = 27;

struct ConvArgs {
  const void* x[3];
  void* y[3];
  const float* w_text;  // [3][C][text_k]
  const float* w_vis;   // [3][C][27]
  int64_t total;        // B*N tokens
  int64_t N, L;
  int C, text_k;
  int T, Hg, Wg, pt;
};

template <typename T> struct Vec8;
template <> struct Vec8<__nv_bfloat16> {
  static __device__ __forceinline__ void load(const __nv_bfloat16* p, float (&v)[8]) {
    uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
  static __device__ __forceinline__ void store(__nv_bfloat16* p, const float (&v)[8]) {
    uint4 u;
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
      w[i] = *reinterpret_cast<uint32_t*>(&h);
    }
    u.x = w[0]; u.y = w[1]; u.z = w[2]; u.w = w[3];
    *reinterpret_cast<uint4*>(p) = u;
  }
};
template <> struct Vec8<float> {
  static __device__ __forceinline__ void load(const float* p, float (&v)[8]) {
    float4 a = __ldg(reinterpret_cast<const float4*>(p));
    float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
  static __device__ __forceinline__ void store(float* p, const float (&v)[8]) {
    reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
  }
};

template <> struct Vec8<__half> {
  static __device__ __forceinline__ void store(__half* p, const float (&v)[8]) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __half2 h = __floats2half2_rn(v[2 * i], v[2 * i + 1]);
      w[i] = *reinterpret_cast<uint32_t*>(&h);
    }
    *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
  }
};

template <typename T, typename TOut>
__global__ void __launch_bounds__(256) shortconv_kernel(ConvArgs a) {
  __shared__ __align__(16) float wv[kVisTaps][kChanPerBlock];
  __shared__ __align__(16) float wt[kMaxTextK][kChanPerBlock];
  const int tensor = blockIdx.z;
  const int cb = blockIdx.y * kChanPerBlock;
  const int C = a.C;
  for (int i = threadIdx.x; i < kChanPerBlock * kVisTaps; i += blockDim.x) {
    const int c = i / kVisTaps, tap = i % kVisTaps;
    wv[tap][c] = (cb + c < C) ? a.w_vis[((int64_t)tensor * C + cb + c) * kVisTaps + tap] : 0.f;
  }
  for (int i = threadIdx.x; i < kChanPerBlock * a.text_k; i += blockDim.x) {
    const int c = i / a.text_k, j = i % a.text_k;
    wt[j][c] = (cb + c < C) ? a.w_text[((int64_t)tensor * C + cb + c) * a.text_k + j] : 0.f;
  }
  __syncthreads();

  const T* __restrict__ x = static_cast<const T*>(a.x[tensor]);
  TOut* __restrict__ y = static_cast<TOut*>(a.y[tensor]);
  const int lane = threadIdx.x & 31;
  const int cl = lane * 8;  // channel offset within the block
  const int c0 = cb + cl;
  if (c0 >= C) return;
  const int64_t tok0 = (int64_t)blockIdx.x * kTokPerBlock;
  const int64_t tok1 = min(tok0 + kTokPerBlock, a.total);
  const int64_t HW = (int64_t)a.Hg * a.Wg;

  for (int64_t it = tok0 + (threadIdx.x >> 5); it < tok1; it += (blockDim.x >> 5)) {
    const int64_t b = it / a.N, n = it - b * a.N;
    const T* xb = x + b * a.N * C;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
    if (n < a.L) {
      for (int j = 0; j < a.text_k; ++j) {
        const int64_t src = n - (a.text_k - 1) + j;
        if (src < 0) continue;
        float v[8];
        Vec8<T>::load(xb + src * C + c0, v);
        const float4 w0 = *reinterpret_cast<const float4*>(&wt[j][cl]);
        const float4 w1 = *reinterpret_cast<const float4*>(&wt[j][cl + 4]);
        acc[0] += w0.x * v[0]; acc[1] += w0.y * v[1]; acc[2] += w0.z * v[2]; acc[3] += w0.w * v[3];
        acc[4] += w1.x * v[4]; acc[5] += w1.y * v[5]; acc[6] += w1.z * v[6]; acc[7] += w1.w * v[7];
      }
    } else {
      const int64_t p = n - a.L;
      const int tt = (int)(p / HW);
      const int rem = (int)(p - (int64_t)tt * HW);
      const int hh = rem / a.Wg, ww = rem - hh * a.Wg;
#pragma unroll
      for (int ta = 0; ta < 3; ++ta) {
        const int t2 = tt + ta - a.pt;
        if (t2 < 0 || t2 >= a.T) continue;
#pragma unroll
        for (int tb = 0; tb < 3; ++tb) {
          const int h2 = hh + tb - 1;
          if (h2 < 0 || h2 >= a.Hg) continue;
#pragma unroll
          for (int te = 0; te < 3; ++te) {
            const int w2 = ww + te - 1;
            if (w2 < 0 || w2 >= a.Wg) continue;
            const int64_t src = a.L + (int64_t)t2 * HW + (int64_t)h2 * a.Wg + w2;
            float v[8];
            Vec8<T>::load(xb + src * C + c0, v);
            const int tap = (ta * 3 + tb) * 3 + te;
            const float4 w0 = *reinterpret_cast<const float4*>(&wv[tap][cl]);
            const float4 w1 = *reinterpret_cast<const float4*>(&wv[tap][cl + 4]);
            acc[0] += w0.x * v[0]; acc[1] += w0.y * v[1]; acc[2] += w0.z * v[2]; acc[3] += w0.w * v[3];
            acc[4] += w1.x * v[4]; acc[5] += w1.y * v[5]; acc[6] += w1.z * v[6]; acc[7] += w1.w * v[7];
          }
        }
      }
    }
    Vec8<TOut>::store(y + b * a.N * C + n * C + c0, acc);
  }
}

}  // namespace

cudaError_t launch_shortconv(const Dims& d, kda_dtype dt, const void* q, const void* k, const void* v,
                             const float* w_text, const float* w_vis, void* qo, void* ko, void* vo,
                             cudaStream_t s, int* launches, bool out_f16) {
  ConvArgs a;
  a.x[0] = q; a.x[1] = k; a.x[2] = v;
  a.y[0] = qo; a.y[1] = ko; a.y[2] = vo;
  a.w_text = w_text; a.w_vis = w_vis;
  a.total = (int64_t)d.B * d.N;
  a.N = d.N; a.L = d.L;
  a.C = d.H * d.dk;
  a.text_k = d.text_k;
  a.T = d.T; a.Hg = d.Hg; a.Wg = d.Wg; a.pt = d.pt;
  if (a.total == 0) return cudaSuccess;
  dim3 grid((unsigned)((a.total + kTokPerBlock - 1) / kTokPerBlock),
            (unsigned)((a.C + kChanPerBlock - 1) / kChanPerBlock), 3);
  if (dt == KDA_DT_BF16 && out_f16) shortconv_kernel<__nv_bfloat16, __half><<<grid, 256, 0, s>>>(a);
  else if (dt == KDA_DT_BF16) shortconv_kernel<__nv_bfloat16, __nv_bfloat16><<<grid, 256, 0, s>>>(a);
  else shortconv_kernel<float, float><<<grid, 256, 0, s>>>(a);
  if (launches) ++*launches;
  return cudaGetLastError();
}

}  // namespace kda
