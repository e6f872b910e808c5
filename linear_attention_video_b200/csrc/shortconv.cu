// Modality-aware depthwise short convolution on q, k and v.
//
// Text tokens: causal 1D depthwise conv; visual tokens: depthwise 3D conv over
// the (T, H, W) latent grid, zero outside the grid, per modality (genai-atlas,
// "How it works"; paper.rainbus.top, section 核心方法).  fp32 accumulation,
// one rounding to the output type, except where the visual conv writes the fp16
// inputs of the tensor-core scan: there it runs on packed fp16 FMAs
// (vis_conv_h2_kernel, below).
//
// Visual part (the bulk of the work, bound by the fp32 FMA pipe): a CTA of two
// warps owns 32 channels of one tensor (one per lane) and a tile of TH = 2 grid
// rows x one run of RUN columns (13 on 52-wide grids, 16 on 64- and 256-wide
// ones), and slides through time; eight CTAs are resident per SM.  Input planes
// (the tile plus a one-pixel halo, zero outside the grid) are copied as they are
// by cp.async into a ring of NSLOT = 3 shared-memory slots, two planes ahead of
// the one being computed.  Each plane is read from shared memory once: a thread
// owns one output row of the run and keeps the partial sums of the three output
// frames that plane feeds (t = f + pt - a for temporal tap a) in registers, so
// every value it reads feeds up to 27 taps.  The frame whose last tap arrived is
// written out and its registers start the frame three ahead.
//
// Text part: a small kernel, one thread per (token, 8 channels).
#include <cuda_fp16.h>

#include <type_traits>


#include "common.cuh"

namespace kda {
namespace {

constexpr int kVisTaps = 27;
constexpr int CG = 32;            // channels per CTA, one per lane
// Small CTAs (two warps) with eight resident per SM measured fastest: 124
// registers a thread keeps one row of three frames in flight, and many small
// tiles hide the plane loads better than a few large ones.
constexpr int TH = 2;             // tile rows
constexpr int RPT = 1;            // output rows per thread
constexpr int NRUN = 1;           // runs per tile row
constexpr int kMinBlocks = 8;     // resident CTAs per SM the register budget is sized for
constexpr int kThreads = 32 * (TH / RPT) * NRUN;   // a warp: 32 channels x one run of RPT rows
constexpr int PH = TH + 2;        // plane rows incl. halo

struct ConvArgs {
  const void* x[3];
  void* y[3];
  const float* w_text;  // [3][C][text_k]
  const float* w_vis;   // [3][C][27]
  int64_t N, L;
  int B, C, text_k;
  int T, Hg, Wg, pt;
  int n_wtiles, n_hbands;
  float* dw_vis;        // [3][C][27], accumulated (weight-gradient kernel only)
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

// store one channel
template <typename T> __device__ __forceinline__ void store1(T* p, float a);
template <> __device__ __forceinline__ void store1<__nv_bfloat16>(__nv_bfloat16* p, float a) { *p = __float2bfloat16_rn(a); }
template <> __device__ __forceinline__ void store1<__half>(__half* p, float a) { *p = __float2half_rn(a); }
template <> __device__ __forceinline__ void store1<float>(float* p, float a) { *p = a; }

// ---- visual kernel -----------------------------------------------------------
// RUN: pixels per thread along a row (compile-time, so the FMA loop carries no
// predicates); a tile is NRUN runs wide.  Columns past the grid edge read the
// zero padding of the plane and their outputs are not stored.  PT: temporal
// offset of the first tap (1 centred, 2 causal, 0 anti-causal: the transpose of
// the causal conv).  FLIP reverses the 27 taps, which turns the kernel into the
// transpose of the conv with the unflipped taps and offset 2 - PT.
constexpr int NSLOT = 3;   // plane slots in shared memory (2 planes in flight)

__device__ __forceinline__ float widen1(__nv_bfloat16 h) { return __bfloat162float(h); }
__device__ __forceinline__ float widen1(float v) { return v; }

// 16-byte cp.async that reads `src_bytes` (16 or 0: zero fill) from global memory
__device__ __forceinline__ void cp_async16_zfill(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" :: "r"(dst), "l"(src), "r"(src_bytes) : "memory");
}

template <typename TIn, int RUN>
struct VisPlane {
  static constexpr int PWr = NRUN * RUN + 2;                       // plane columns incl. halo
  static constexpr int PIX_CHUNKS = CG * (int)sizeof(TIn) / 16;    // 16-byte chunks per pixel
  static constexpr int NCHUNK = PH * PWr * PIX_CHUNKS;
  static constexpr int NPF = (NCHUNK + kThreads - 1) / kThreads;   // chunks per thread
  static constexpr int BYTES = PH * PWr * CG * (int)sizeof(TIn);
};

// One plane f: FMAs into the three frames it feeds (RPT output rows each), then
// the completed frame out.  Plane row ir feeds output row orow through tap
// tb = ir - orow.
template <typename TIn, typename TOut, int RUN, int PT>
__device__ __forceinline__ void vis_plane_step(const TIn* pl, bool compute, const float (&wv)[kVisTaps],
                                               float (&an)[RPT][RUN], float (&ac)[RPT][RUN], float (&ap)[RPT][RUN],
                                               TOut* yo, int64_t row_stride, bool emit, int nrow, int nrun,
                                               int64_t C) {
  constexpr int PWr = VisPlane<TIn, RUN>::PWr;
  if (compute) {
#pragma unroll
    for (int ir = 0; ir < RPT + 2; ++ir) {
      const TIn* src = pl + ir * PWr * CG;
      float in[RUN + 2];
#pragma unroll
      for (int i = 0; i < RUN + 2; ++i) in[i] = widen1(src[i * CG]);
#pragma unroll
      for (int orow = 0; orow < RPT; ++orow) {
        const int tb = ir - orow;
        if (tb < 0 || tb > 2) continue;
#pragma unroll
        for (int te = 0; te < 3; ++te) {
          const float c0 = wv[tb * 3 + te], c1 = wv[9 + tb * 3 + te], c2 = wv[18 + tb * 3 + te];
#pragma unroll
          for (int i = 0; i < RUN; ++i) {
            an[orow][i] = fmaf(c0, in[i + te], an[orow][i]);
            ac[orow][i] = fmaf(c1, in[i + te], ac[orow][i]);
            ap[orow][i] = fmaf(c2, in[i + te], ap[orow][i]);
          }
        }
      }
    }
  }
#pragma unroll
  for (int orow = 0; orow < RPT; ++orow) {
    if (emit && orow < nrow) {
#pragma unroll
      for (int i = 0; i < RUN; ++i)
        if (i < nrun) store1<TOut>(yo + orow * row_stride + (int64_t)i * C, ap[orow][i]);
    }
#pragma unroll
    for (int i = 0; i < RUN; ++i) ap[orow][i] = 0.f;   // ap becomes the frame three ahead
  }
}

template <typename TIn, typename TOut, int RUN, int PT, bool FLIP>
__global__ void __launch_bounds__(kThreads, kMinBlocks) vis_conv_kernel(ConvArgs a) {
  using VP = VisPlane<TIn, RUN>;
  constexpr int PWr = VP::PWr;
  extern __shared__ __align__(128) uint8_t slots[];   // [NSLOT][PH][PWr][CG] of TIn
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int tile = blockIdx.x;
  const int wt = tile % a.n_wtiles, hb = tile / a.n_wtiles;
  const int cg0 = blockIdx.y * CG;
  const int tensor = blockIdx.z % 3, b = blockIdx.z / 3;
  const int C = a.C;
  const int tw0 = wt * (NRUN * RUN), th0 = hb * TH;
  const int TW = min(NRUN * RUN, a.Wg - tw0), THh = min(TH, a.Hg - th0);
  const int64_t HW = (int64_t)a.Hg * a.Wg;
  // pointers chosen by selects, so the argument block is not copied to local memory
  const void* xs = tensor == 0 ? a.x[0] : (tensor == 1 ? a.x[1] : a.x[2]);
  void* ys = tensor == 0 ? a.y[0] : (tensor == 1 ? a.y[1] : a.y[2]);
  const TIn* x = static_cast<const TIn*>(xs) + ((int64_t)b * a.N + a.L) * C + cg0;
  TOut* y = static_cast<TOut*>(ys) + ((int64_t)b * a.N + a.L) * C + cg0;

  const int row = RPT * (warp % (TH / RPT)), run = warp / (TH / RPT);   // output rows row .. row + RPT - 1
  const int w0 = run * RUN;
  const int nrun = max(0, min(RUN, TW - w0));
  const int nrow = nrun > 0 ? max(0, min(RPT, THh - row)) : 0;   // rows of this thread inside the grid
  const bool active = nrow > 0;

  float wv[kVisTaps];
  {
    const float* wbase = a.w_vis + ((int64_t)tensor * C + cg0 + lane) * kVisTaps;
#pragma unroll
    for (int i = 0; i < kVisTaps; ++i) wv[i] = wbase[FLIP ? kVisTaps - 1 - i : i];
  }

  // this thread's chunks of a plane: element offset inside a frame (-1: outside the grid)
  int goff[VP::NPF];
#pragma unroll
  for (int i = 0; i < VP::NPF; ++i) {
    const int e = tid + i * kThreads;
    goff[i] = -2;   // beyond the plane: nothing to copy
    if (e < VP::NCHUNK) {
      const int cb = e % VP::PIX_CHUNKS, pix = e / VP::PIX_CHUNKS;
      const int pr = pix / PWr, pc = pix - pr * PWr;
      const int hh = th0 + pr - 1, ww = tw0 + pc - 1;
      goff[i] = (hh >= 0 && hh < a.Hg && ww >= 0 && ww < a.Wg)
                    ? (hh * a.Wg + ww) * C + cb * (16 / (int)sizeof(TIn)) : -1;
    }
  }
  const uint32_t slot0 = (uint32_t)__cvta_generic_to_shared(slots);
  auto issue = [&](int f) {   // plane f -> slot f % NSLOT, one commit group per call
    if (f < a.T) {
      const TIn* xf = x + (int64_t)f * HW * C;
      const uint32_t dst = slot0 + (uint32_t)(f % NSLOT) * VP::BYTES;
#pragma unroll
      for (int i = 0; i < VP::NPF; ++i) {
        if (goff[i] >= -1)
          cp_async16_zfill(dst + (uint32_t)(tid + i * kThreads) * 16u, goff[i] >= 0 ? xf + goff[i] : x,
                           goff[i] >= 0 ? 16u : 0u);
      }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };

  float s0[RPT][RUN], s1[RPT][RUN], s2[RPT][RUN];
#pragma unroll
  for (int r = 0; r < RPT; ++r)
#pragma unroll
    for (int i = 0; i < RUN; ++i) { s0[r][i] = 0.f; s1[r][i] = 0.f; s2[r][i] = 0.f; }
  for (int f = 0; f < NSLOT - 1; ++f) issue(f);

  // after plane f, frame f+PT-2 is complete; 2 - PT steps past the last plane
  // (no data) flush the frames up to T-1
  const int f_end = a.T + 2 - PT;
  const TIn* pl_base = reinterpret_cast<const TIn*>(slots) + (row * PWr + w0) * CG + lane;
  TOut* y_base = y + ((int64_t)(th0 + row) * a.Wg + tw0 + w0) * C + lane;
  auto step = [&](int f, float (&an)[RPT][RUN], float (&ac)[RPT][RUN], float (&ap)[RPT][RUN]) {
    asm volatile("cp.async.wait_group %0;" :: "n"(NSLOT - 2) : "memory");
    __syncthreads();   // plane f in place everywhere; slot (f-1) % NSLOT no longer read
    issue(f + NSLOT - 1);
    const int t = f + PT - 2;
    const bool tv = t >= 0 && t < a.T;
    vis_plane_step<TIn, TOut, RUN, PT>(pl_base + (f % NSLOT) * (VP::BYTES / (int)sizeof(TIn)),
                                       active && f < a.T, wv, an, ac, ap, y_base + (int64_t)t * HW * C,
                                       (int64_t)a.Wg * C, active && tv, nrow, nrun, C);
  };
  // roles rotate with f % 3: (frame f+PT, f+PT-1, f+PT-2) live in sets ((f+PT)%3, ...)
  for (int f = 0; f < f_end; f += 3) {
    if (PT == 1) {
      step(f, s1, s0, s2);
      if (f + 1 < f_end) step(f + 1, s2, s1, s0);
      if (f + 2 < f_end) step(f + 2, s0, s2, s1);
    } else if (PT == 2) {
      step(f, s2, s1, s0);
      if (f + 1 < f_end) step(f + 1, s0, s2, s1);
      if (f + 2 < f_end) step(f + 2, s1, s0, s2);
    } else {
      step(f, s0, s2, s1);
      if (f + 1 < f_end) step(f + 1, s1, s0, s2);
      if (f + 2 < f_end) step(f + 2, s2, s1, s0);
    }
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
}

// ---- visual kernel on packed fp16 (bf16 inputs, fp16 outputs) ------------------------
// The conv feeding the tensor-core scan, whose operands are fp16: the same tiles, plane ring and
// frame rotation as vis_conv_kernel, but a lane owns two adjacent channels (a CTA 64) and every
// tap is one fma.rn.f16x2 over both, accumulating in fp16.  That halves the FMA instructions of
// the issue-bound fp32 kernel; the outputs carry a relative error of about 8e-4 (27 fp16
// roundings) instead of 2e-4 (one rounding of an fp32 sum), the size of the scan's own fp16
// operand roundings.
constexpr int CG2 = 64;   // channels per CTA: two per lane

template <int RUN>
struct VisPlaneH2 {
  static constexpr int PWr = NRUN * RUN + 2;
  static constexpr int WPP = CG2 / 2;                   // 32-bit words (channel pairs) per pixel
  static constexpr int PIX_CHUNKS = CG2 * 2 / 16;       // 16-byte chunks per pixel
  static constexpr int NCHUNK = PH * PWr * PIX_CHUNKS;
  static constexpr int NPF = (NCHUNK + kThreads - 1) / kThreads;
  static constexpr int BYTES = PH * PWr * CG2 * 2;
};

// two bf16 (one 32-bit word) -> fp16 pair
__device__ __forceinline__ __half2 bf2_to_h2(uint32_t u) {
  return __floats2half2_rn(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
}

template <int RUN>
__device__ __forceinline__ void vis_plane_step_h2(const uint32_t* pl, bool compute, const __half2 (&wv)[kVisTaps],
                                                  __half2 (&an)[RUN], __half2 (&ac)[RUN], __half2 (&ap)[RUN],
                                                  __half* yo, bool emit, int nrun, int64_t C) {
  constexpr int PWr = VisPlaneH2<RUN>::PWr, WPP = VisPlaneH2<RUN>::WPP;
  if (compute) {
#pragma unroll
    for (int tb = 0; tb < 3; ++tb) {   // plane row tb feeds the thread's output row through tap row tb
      const uint32_t* src = pl + tb * PWr * WPP;
      __half2 in[RUN + 2];
#pragma unroll
      for (int i = 0; i < RUN + 2; ++i) in[i] = bf2_to_h2(src[i * WPP]);
#pragma unroll
      for (int te = 0; te < 3; ++te) {
        const __half2 c0 = wv[tb * 3 + te], c1 = wv[9 + tb * 3 + te], c2 = wv[18 + tb * 3 + te];
#pragma unroll
        for (int i = 0; i < RUN; ++i) {
          an[i] = __hfma2(c0, in[i + te], an[i]);
          ac[i] = __hfma2(c1, in[i + te], ac[i]);
          ap[i] = __hfma2(c2, in[i + te], ap[i]);
        }
      }
    }
  }
  if (emit) {
#pragma unroll
    for (int i = 0; i < RUN; ++i)
      if (i < nrun) *reinterpret_cast<__half2*>(yo + (int64_t)i * C) = ap[i];
  }
#pragma unroll
  for (int i = 0; i < RUN; ++i) ap[i] = __float2half2_rn(0.f);   // ap becomes the frame three ahead
}

// The text tokens of one (64-channel group, tensor, batch item) in a CTA of the packed visual
// launch: the causal 1D conv of text_conv_kernel (fp32 accumulation, one rounding to fp16), a lane
// owning two channels and each warp half of the tokens.  These CTAs run beside the visual tiles.
__device__ __noinline__ void text_part_h2(const ConvArgs& a, const void* xs, void* ys, int cg0, int tensor, int b) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int C = a.C, K = a.text_k, c = cg0 + 2 * lane;
  const uint32_t* x = reinterpret_cast<const uint32_t*>(static_cast<const __nv_bfloat16*>(xs) + (int64_t)b * a.N * C + c);
  __half* y = static_cast<__half*>(ys) + (int64_t)b * a.N * C + c;
  const float* w = a.w_text + ((int64_t)tensor * C + c) * K;
  float w0[8], w1[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    w0[j] = j < K ? w[j] : 0.f;
    w1[j] = j < K ? w[K + j] : 0.f;
  }
  const int64_t per = (a.L + 1) / 2, n0 = warp * per, n1 = min(a.L, n0 + per);
  for (int64_t n = n0; n < n1; ++n) {
    float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int64_t src = n - (K - 1) + j;
      if (j < K && src >= 0) {
        const uint32_t u = __ldg(x + src * (C / 2));
        acc0 = fmaf(w0[j], __uint_as_float(u << 16), acc0);
        acc1 = fmaf(w1[j], __uint_as_float(u & 0xffff0000u), acc1);
      }
    }
    *reinterpret_cast<__half2*>(y + n * C) = __floats2half2_rn(acc0, acc1);
  }
}

template <int RUN, int PT>
__global__ void __launch_bounds__(kThreads, kMinBlocks) vis_conv_h2_kernel(ConvArgs a) {
  static_assert(RPT == 1, "one output row per thread");
  using VP = VisPlaneH2<RUN>;
  constexpr int PWr = VP::PWr;
  extern __shared__ __align__(128) uint8_t slots[];   // [NSLOT][PH][PWr][CG2] of bf16
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int tile = blockIdx.x;
  const int wt = tile % a.n_wtiles, hb = tile / a.n_wtiles;
  const int cg0 = blockIdx.y * CG2;
  const int tensor = blockIdx.z % 3, b = blockIdx.z / 3;
  const int C = a.C;
  const int tw0 = wt * (NRUN * RUN), th0 = hb * TH;
  const int TW = min(NRUN * RUN, a.Wg - tw0), THh = min(TH, a.Hg - th0);
  const int64_t HW = (int64_t)a.Hg * a.Wg;
  const void* xs = tensor == 0 ? a.x[0] : (tensor == 1 ? a.x[1] : a.x[2]);
  void* ys = tensor == 0 ? a.y[0] : (tensor == 1 ? a.y[1] : a.y[2]);
  if (tile >= a.n_wtiles * a.n_hbands) {   // past the visual tiles: the text tokens
    text_part_h2(a, xs, ys, cg0, tensor, b);
    return;
  }
  const __nv_bfloat16* x = static_cast<const __nv_bfloat16*>(xs) + ((int64_t)b * a.N + a.L) * C + cg0;
  __half* y = static_cast<__half*>(ys) + ((int64_t)b * a.N + a.L) * C + cg0;

  const int row = warp % TH, run = warp / TH;
  const int w0 = run * RUN;
  const int nrun = max(0, min(RUN, TW - w0));
  const bool active = nrun > 0 && row < THh;

  __half2 wv[kVisTaps];
  {
    const float* w0p = a.w_vis + ((int64_t)tensor * C + cg0 + 2 * lane) * kVisTaps;
#pragma unroll
    for (int i = 0; i < kVisTaps; ++i) wv[i] = __floats2half2_rn(w0p[i], w0p[kVisTaps + i]);
  }

  int goff[VP::NPF];
#pragma unroll
  for (int i = 0; i < VP::NPF; ++i) {
    const int e = tid + i * kThreads;
    goff[i] = -2;
    if (e < VP::NCHUNK) {
      const int cb = e % VP::PIX_CHUNKS, pix = e / VP::PIX_CHUNKS;
      const int pr = pix / PWr, pc = pix - pr * PWr;
      const int hh = th0 + pr - 1, ww = tw0 + pc - 1;
      goff[i] = (hh >= 0 && hh < a.Hg && ww >= 0 && ww < a.Wg) ? (hh * a.Wg + ww) * C + cb * 8 : -1;
    }
  }
  const uint32_t slot0 = (uint32_t)__cvta_generic_to_shared(slots);
  auto issue = [&](int f) {
    if (f < a.T) {
      const __nv_bfloat16* xf = x + (int64_t)f * HW * C;
      const uint32_t dst = slot0 + (uint32_t)(f % NSLOT) * VP::BYTES;
#pragma unroll
      for (int i = 0; i < VP::NPF; ++i) {
        if (goff[i] >= -1)
          cp_async16_zfill(dst + (uint32_t)(tid + i * kThreads) * 16u, goff[i] >= 0 ? xf + goff[i] : x,
                           goff[i] >= 0 ? 16u : 0u);
      }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };

  __half2 s0[RUN], s1[RUN], s2[RUN];
#pragma unroll
  for (int i = 0; i < RUN; ++i) { s0[i] = __float2half2_rn(0.f); s1[i] = s0[i]; s2[i] = s0[i]; }
  for (int f = 0; f < NSLOT - 1; ++f) issue(f);

  const int f_end = a.T + 2 - PT;
  const uint32_t* pl_base = reinterpret_cast<const uint32_t*>(slots) + (row * PWr + w0) * VP::WPP + lane;
  __half* y_base = y + ((int64_t)(th0 + row) * a.Wg + tw0 + w0) * C + 2 * lane;
  auto step = [&](int f, __half2 (&an)[RUN], __half2 (&ac)[RUN], __half2 (&ap)[RUN]) {
    asm volatile("cp.async.wait_group %0;" :: "n"(NSLOT - 2) : "memory");
    __syncthreads();
    issue(f + NSLOT - 1);
    const int t = f + PT - 2;
    const bool tv = t >= 0 && t < a.T;
    vis_plane_step_h2<RUN>(pl_base + (f % NSLOT) * (VP::BYTES / 4), active && f < a.T, wv, an, ac, ap,
                           y_base + (int64_t)t * HW * C, active && tv, nrun, C);
  };
  for (int f = 0; f < f_end; f += 3) {
    if (PT == 1) {
      step(f, s1, s0, s2);
      if (f + 1 < f_end) step(f + 1, s2, s1, s0);
      if (f + 2 < f_end) step(f + 2, s0, s2, s1);
    } else {
      step(f, s2, s1, s0);
      if (f + 1 < f_end) step(f + 1, s0, s2, s1);
      if (f + 2 < f_end) step(f + 2, s1, s0, s2);
    }
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
}

// ---- visual weight gradient ------------------------------------------------------
// dw[c][a][b][e] = sum over t, h, w of dy[t, h, w, c] x[t + a - PT, h + b - 1, w + e - 1, c].
// Same tiles and plane ring as the forward kernel: plane f of x meets the dy frames
// f + PT - a (a = 0, 1, 2) of the thread's pixels, which sit in three register sets
// rotating like the forward's accumulators (the next frame is loaded into the set
// just used, so its latency overlaps the next barrier).  Each thread sums the 27 taps
// of its channel over its pixels; the CTA's warps meet in shared memory and add
// their totals to dw with one atomic per (channel, tap).
template <typename TIn, int RUN, int PT>
__global__ void __launch_bounds__(kThreads, kMinBlocks) vis_dw_kernel(ConvArgs a) {
  using VP = VisPlane<TIn, RUN>;
  constexpr int PWr = VP::PWr;
  constexpr int NW = kThreads / 32;
  extern __shared__ __align__(128) uint8_t slots[];   // [NSLOT][PH][PWr][CG] of TIn
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int tile = blockIdx.x;
  const int wt = tile % a.n_wtiles, hb = tile / a.n_wtiles;
  const int cg0 = blockIdx.y * CG;
  const int tensor = blockIdx.z % 3, b = blockIdx.z / 3;
  const int C = a.C;
  const int tw0 = wt * (NRUN * RUN), th0 = hb * TH;
  const int TW = min(NRUN * RUN, a.Wg - tw0), THh = min(TH, a.Hg - th0);
  const int64_t HW = (int64_t)a.Hg * a.Wg;
  const void* xs = tensor == 0 ? a.x[0] : (tensor == 1 ? a.x[1] : a.x[2]);
  const void* ys = tensor == 0 ? a.y[0] : (tensor == 1 ? a.y[1] : a.y[2]);
  const TIn* x = static_cast<const TIn*>(xs) + ((int64_t)b * a.N + a.L) * C + cg0;
  const float* dy = static_cast<const float*>(ys) + ((int64_t)b * a.N + a.L) * C + cg0;

  const int row = RPT * (warp % (TH / RPT)), run = warp / (TH / RPT);
  const int w0 = run * RUN;
  const int nrun = max(0, min(RUN, TW - w0));
  const int nrow = nrun > 0 ? max(0, min(RPT, THh - row)) : 0;

  int goff[VP::NPF];
#pragma unroll
  for (int i = 0; i < VP::NPF; ++i) {
    const int e = tid + i * kThreads;
    goff[i] = -2;
    if (e < VP::NCHUNK) {
      const int cb = e % VP::PIX_CHUNKS, pix = e / VP::PIX_CHUNKS;
      const int pr = pix / PWr, pc = pix - pr * PWr;
      const int hh = th0 + pr - 1, ww = tw0 + pc - 1;
      goff[i] = (hh >= 0 && hh < a.Hg && ww >= 0 && ww < a.Wg)
                    ? (hh * a.Wg + ww) * C + cb * (16 / (int)sizeof(TIn)) : -1;
    }
  }
  const uint32_t slot0 = (uint32_t)__cvta_generic_to_shared(slots);
  auto issue = [&](int f) {
    if (f < a.T) {
      const TIn* xf = x + (int64_t)f * HW * C;
      const uint32_t dst = slot0 + (uint32_t)(f % NSLOT) * VP::BYTES;
#pragma unroll
      for (int i = 0; i < VP::NPF; ++i) {
        if (goff[i] >= -1)
          cp_async16_zfill(dst + (uint32_t)(tid + i * kThreads) * 16u, goff[i] >= 0 ? xf + goff[i] : x,
                           goff[i] >= 0 ? 16u : 0u);
      }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };

  const float* dy_base = dy + ((int64_t)(th0 + row) * a.Wg + tw0 + w0) * C + lane;
  auto load_dy = [&](int t, float (&d)[RPT][RUN]) {   // frame t of this thread's pixels, zero outside
    const bool tv = t >= 0 && t < a.T;
#pragma unroll
    for (int r = 0; r < RPT; ++r)
#pragma unroll
      for (int i = 0; i < RUN; ++i)
        d[r][i] = (tv && r < nrow && i < nrun) ? dy_base[(int64_t)t * HW * C + ((int64_t)r * a.Wg + i) * C] : 0.f;
  };
  float acc[kVisTaps];
#pragma unroll
  for (int i = 0; i < kVisTaps; ++i) acc[i] = 0.f;
  float s0[RPT][RUN], s1[RPT][RUN], s2[RPT][RUN];
  // frame X of dy lives in set (X + 3) % 3; before plane 0: frames PT - 2, PT - 1, PT
  if (PT == 1) { load_dy(-1, s2); load_dy(0, s0); load_dy(1, s1); }
  else if (PT == 2) { load_dy(0, s0); load_dy(1, s1); load_dy(2, s2); }
  else { load_dy(-2, s1); load_dy(-1, s2); load_dy(0, s0); }
  for (int f = 0; f < NSLOT - 1; ++f) issue(f);

  const TIn* pl_base = reinterpret_cast<const TIn*>(slots) + (row * PWr + w0) * CG + lane;
  const bool active = nrow > 0;
  // plane f with the dy frames f + PT (d0), f + PT - 1 (d1), f + PT - 2 (d2); then frame
  // f + PT + 1 replaces d2
  auto step = [&](int f, float (&d0)[RPT][RUN], float (&d1)[RPT][RUN], float (&d2)[RPT][RUN]) {
    asm volatile("cp.async.wait_group %0;" :: "n"(NSLOT - 2) : "memory");
    __syncthreads();
    issue(f + NSLOT - 1);
    if (active) {
      const TIn* pl = pl_base + (f % NSLOT) * (VP::BYTES / (int)sizeof(TIn));
#pragma unroll
      for (int ir = 0; ir < RPT + 2; ++ir) {
        const TIn* src = pl + ir * PWr * CG;
        float in[RUN + 2];
#pragma unroll
        for (int i = 0; i < RUN + 2; ++i) in[i] = widen1(src[i * CG]);
#pragma unroll
        for (int orow = 0; orow < RPT; ++orow) {
          const int tb = ir - orow;
          if (tb < 0 || tb > 2) continue;
#pragma unroll
          for (int te = 0; te < 3; ++te) {
            float p0 = 0.f, p1 = 0.f, p2 = 0.f;
#pragma unroll
            for (int i = 0; i < RUN; ++i) {
              p0 = fmaf(d0[orow][i], in[i + te], p0);
              p1 = fmaf(d1[orow][i], in[i + te], p1);
              p2 = fmaf(d2[orow][i], in[i + te], p2);
            }
            acc[tb * 3 + te] += p0;
            acc[9 + tb * 3 + te] += p1;
            acc[18 + tb * 3 + te] += p2;
          }
        }
      }
    }
    load_dy(f + PT + 1, d2);
  };
  for (int f = 0; f < a.T; f += 3) {
    if (PT == 1) {
      step(f, s1, s0, s2);
      if (f + 1 < a.T) step(f + 1, s2, s1, s0);
      if (f + 2 < a.T) step(f + 2, s0, s2, s1);
    } else if (PT == 2) {
      step(f, s2, s1, s0);
      if (f + 1 < a.T) step(f + 1, s0, s2, s1);
      if (f + 2 < a.T) step(f + 2, s1, s0, s2);
    } else {
      step(f, s0, s2, s1);
      if (f + 1 < a.T) step(f + 1, s1, s0, s2);
      if (f + 2 < a.T) step(f + 2, s2, s1, s0);
    }
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  __syncthreads();   // the ring is free: the warps' tap sums meet there
  float* red = reinterpret_cast<float*>(slots);   // [NW][27][32]
#pragma unroll
  for (int i = 0; i < kVisTaps; ++i) red[(warp * kVisTaps + i) * 32 + lane] = acc[i];
  __syncthreads();
  for (int i = warp; i < kVisTaps; i += NW) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) s += red[(w * kVisTaps + i) * 32 + lane];
    atomicAdd(a.dw_vis + ((int64_t)tensor * C + cg0 + lane) * kVisTaps + i, s);
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

// MODE 0: the conv; 1: its transpose (taps reversed, offset 2 - pt); 2: the weight gradient
template <typename TIn, typename TOut, int RUN, int PT, int MODE>
cudaError_t launch_vis_pt(const ConvArgs& a, cudaStream_t s) {
  const size_t smem = (size_t)NSLOT * VisPlane<TIn, RUN>::BYTES;
  dim3 grid((unsigned)(a.n_wtiles * a.n_hbands), (unsigned)(a.C / CG), (unsigned)(3 * a.B));
  cudaError_t e;
  if (MODE == 2) {
    static_assert(kThreads / 32 * kVisTaps * 32 * 4 <= NSLOT * VisPlane<__nv_bfloat16, 8>::BYTES,
                  "the tap sums fit in the plane ring");
    e = cudaFuncSetAttribute(vis_dw_kernel<TIn, RUN, PT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    vis_dw_kernel<TIn, RUN, PT><<<grid, kThreads, smem, s>>>(a);
  } else {
    e = cudaFuncSetAttribute(vis_conv_kernel<TIn, TOut, RUN, PT, MODE == 1>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    vis_conv_kernel<TIn, TOut, RUN, PT, MODE == 1><<<grid, kThreads, smem, s>>>(a);
  }
  return cudaGetLastError();
}

template <typename TIn, typename TOut, int RUN, int MODE>
cudaError_t launch_vis(const ConvArgs& a0, cudaStream_t s) {
  ConvArgs a = a0;
  a.n_wtiles = (a.Wg + NRUN * RUN - 1) / (NRUN * RUN);
  if (MODE == 1)   // transpose: centred stays centred, causal becomes anti-causal
    return a.pt == 2 ? launch_vis_pt<TIn, TOut, RUN, 0, MODE>(a, s) : launch_vis_pt<TIn, TOut, RUN, 1, MODE>(a, s);
  return a.pt == 2 ? launch_vis_pt<TIn, TOut, RUN, 2, MODE>(a, s) : launch_vis_pt<TIn, TOut, RUN, 1, MODE>(a, s);
}

// widest run whose tiles cover the row with the least padding
template <typename TIn, typename TOut, int MODE>
cudaError_t launch_vis_any(const ConvArgs& a, cudaStream_t s) {
  if (a.Wg % 52 == 0 || (a.Wg <= 52 && a.Wg > 48)) return launch_vis<TIn, TOut, 13, MODE>(a, s);
  if (a.Wg % 64 == 0 || a.Wg > 52) return launch_vis<TIn, TOut, 16, MODE>(a, s);
  return launch_vis<TIn, TOut, 8, MODE>(a, s);
}

template <int RUN>
cudaError_t launch_vis_h2(const ConvArgs& a0, cudaStream_t s) {
  ConvArgs a = a0;
  a.n_wtiles = (a.Wg + NRUN * RUN - 1) / (NRUN * RUN);
  const size_t smem = (size_t)NSLOT * VisPlaneH2<RUN>::BYTES;
  // one more CTA column for the text tokens, when there are any
  dim3 grid((unsigned)(a.n_wtiles * a.n_hbands + (a.L > 0 ? 1 : 0)), (unsigned)(a.C / CG2), (unsigned)(3 * a.B));
  cudaError_t e;
  if (a.pt == 2) {
    e = cudaFuncSetAttribute(vis_conv_h2_kernel<RUN, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    vis_conv_h2_kernel<RUN, 2><<<grid, kThreads, smem, s>>>(a);
  } else {
    e = cudaFuncSetAttribute(vis_conv_h2_kernel<RUN, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    vis_conv_h2_kernel<RUN, 1><<<grid, kThreads, smem, s>>>(a);
  }
  return cudaGetLastError();
}

template <typename TIn, typename TOut>
cudaError_t launch_t(const ConvArgs& a, cudaStream_t s, int* launches) {
  // the fp16 outputs feed the tensor-core scan: the visual conv runs on packed fp16, its launch
  // doing the text tokens too
  constexpr bool kPackedOut = std::is_same_v<TIn, __nv_bfloat16> && std::is_same_v<TOut, __half>;
  const bool packed = kPackedOut && a.T > 0 && a.C % CG2 == 0;
  if (a.L > 0 && !packed) {
    const int64_t total = (int64_t)a.B * a.L * (a.C / 8);
    text_conv_kernel<TIn, TOut><<<dim3((unsigned)((total + 255) / 256), 3), 256, 0, s>>>(a);
    if (launches) ++*launches;
  }
  if (a.T > 0) {
    if (launches) ++*launches;
    if constexpr (kPackedOut) {
      if (packed) {
        if (a.Wg % 52 == 0 || (a.Wg <= 52 && a.Wg > 48)) return launch_vis_h2<13>(a, s);
        if (a.Wg % 64 == 0 || a.Wg > 52) return launch_vis_h2<16>(a, s);
        return launch_vis_h2<8>(a, s);
      }
    }
    return launch_vis_any<TIn, TOut, 0>(a, s);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_shortconv(const Dims& d, kda_dtype dt, const void* q, const void* k, const void* v,
                             const float* w_text, const float* w_vis, void* qo, void* ko, void* vo,
                             cudaStream_t s, int* launches, bool out_f16, bool out_f32) {
  ConvArgs a;
  a.x[0] = q; a.x[1] = k; a.x[2] = v;
  a.y[0] = qo; a.y[1] = ko; a.y[2] = vo;
  a.w_text = w_text; a.w_vis = w_vis;
  a.N = d.N; a.L = d.L; a.B = d.B;
  a.C = d.H * d.dk;
  a.text_k = d.text_k;
  a.T = d.T; a.Hg = d.Hg; a.Wg = d.Wg; a.pt = d.pt;
  a.n_wtiles = 0;   // set per run length by launch_vis
  a.n_hbands = d.T > 0 ? (d.Hg + TH - 1) / TH : 0;
  if ((int64_t)d.B * d.N == 0) return cudaSuccess;
  cudaError_t e;
  int n = 0;
  if (dt == KDA_DT_BF16 && out_f32) e = launch_t<__nv_bfloat16, float>(a, s, &n);
  else if (dt == KDA_DT_BF16 && out_f16) e = launch_t<__nv_bfloat16, __half>(a, s, &n);
  else if (dt == KDA_DT_BF16) e = launch_t<__nv_bfloat16, __nv_bfloat16>(a, s, &n);
  else e = launch_t<float, float>(a, s, &n);
  if (e == cudaSuccess && launches) *launches += n;
  return e;
}

cudaError_t launch_shortconv_bwd_vis(const Dims& d, kda_dtype dt, const void* const x[3], const float* const dy[3],
                                     void* const dx[3], const float* w_vis, float* dw_vis, cudaStream_t s,
                                     int* launches) {
  if (d.T <= 0 || (int64_t)d.B * d.N == 0) return cudaSuccess;
  ConvArgs a;
  for (int i = 0; i < 3; ++i) { a.x[i] = dy[i]; a.y[i] = dx[i]; }
  a.w_text = nullptr; a.w_vis = w_vis; a.dw_vis = dw_vis;
  a.N = d.N; a.L = d.L; a.B = d.B;
  a.C = d.H * d.dk;
  a.text_k = d.text_k;
  a.T = d.T; a.Hg = d.Hg; a.Wg = d.Wg; a.pt = d.pt;
  a.n_wtiles = 0;
  a.n_hbands = (d.Hg + TH - 1) / TH;
  // dx of the visual tokens: the transposed conv of dy
  cudaError_t e = dt == KDA_DT_BF16 ? launch_vis_any<float, __nv_bfloat16, 1>(a, s) : launch_vis_any<float, float, 1>(a, s);
  if (e != cudaSuccess) return e;
  // dw: the raw inputs against dy
  for (int i = 0; i < 3; ++i) { a.x[i] = x[i]; a.y[i] = const_cast<float*>(dy[i]); }
  e = dt == KDA_DT_BF16 ? launch_vis_any<__nv_bfloat16, float, 2>(a, s) : launch_vis_any<float, float, 2>(a, s);
  if (e == cudaSuccess && launches) *launches += 2;
  return e;
}

}  // namespace kda
