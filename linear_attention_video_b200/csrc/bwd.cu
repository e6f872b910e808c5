// Backward pass of the modality-aware short convolution + KDA scan: the
// gradients of kda_fwd's outputs (o and the final state) with respect to q, k,
// v, log alpha, beta, the conv weights and the initial state, at fp32 accuracy
// (products on the tensor cores as split tf32, see wmma3).
//
// Forward step per head (paper.rainbus.top, section 方法步骤详情, step (5)):
//     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,   o_t = S_t^T q_t.
// The backward runs in the chunked (UT/WY) form over CH-token chunks.  With g
// the running sum of log alpha from the chunk start, gl its last row,
// KG = k e^g, QG = q e^g, Kt = k e^{gl - g}, A = strict-lower(Diag(beta) (k k^T o e^{g_r - g_i})),
// P = lower(q k^T o e^{g_r - g_i}), X = (I + A)^{-1}, T = X Diag(beta), W = T KG:
//     U = T V - W S_in,   O = QG S_in + P U,   S_out = Diag(e^{gl}) S_in + Kt^T U.
// Its adjoint, chunk by chunk in reverse with dS the gradient reaching S_out:
//     dU = P^T dO + Kt dS,   dS_in = Diag(e^{gl}) dS + QG^T dO - W^T dU,
// then the chain rule through U, O, S_out, T, A, P and the exponential factors
// gives the chunk's dq, dk, dv, dlog alpha and dbeta (no term crosses the
// chunk boundary except dS).  The pairwise decays e^{g_r - g_i} are split as
// e^{g_r - g_m} e^{g_m - g_i} around g_m, the running sum at token CH/2 - 1;
// a chunk whose |g - g_m| exceeds kRange nats sets KDA_ERR_RANGE.
//
// Kernels, in launch order:
//   conv (forward, fp32 out)   q', k', v' recomputed from the raw inputs
//   cbwd_prep_kernel           per chunk: W, U~ = T V, Kt, X, A/beta, e^{gl}, and
//                              the dO terms Z = P^T dO, Y = QG^T dO
//   cbwd_chain_kernel<D, false>  per CW value columns: S_in of every chunk, U
//   cbwd_chain_kernel<D, true>   per CW value columns, in reverse: dS of every chunk, dU, dS0
//                              (fp32 problems; bf16 problems run both chains as one launch of
//                              cbwd_chain_h_kernel, on fp16 operands)
//   cbwd_state_grad_kernel     per chunk: the contractions with S_in and dS
//                              (dQG, dW, dKt), dP, dU V^T
//   cbwd_local_grad_kernel     per chunk: dT, the inverse's adjoint, dq, dk, dv,
//                              dlog alpha, dbeta
//   bwd_beta_kernel            dbeta fp32 -> dtype
//   conv_bwd_dx_kernel         text tokens: dx = transpose of the causal 1D conv
//   conv_bwd_dw_kernel         text tokens: dw = sum over tokens of x * dy per tap
//   vis_conv_kernel (FLIP)     visual tokens: dx = the conv with reversed taps
//   vis_dw_kernel              visual tokens: dw, on the forward conv's tiles
#include "common.cuh"

#include <cuda_fp16.h>

namespace kda {
namespace {

constexpr int CH = 64;          // tokens per chunk
constexpr int NT = 256;         // threads of every scan kernel: a 16 x 16 grid (ty, tx)
constexpr int LDC = CH + 4;     // row stride of CH x CH tiles in shared memory (4 mod 32, see wmma3)
constexpr int CW = 16;          // value columns per CTA of the two chains
constexpr int JB = 32;          // value columns per stage of the state-gradient kernel
constexpr int LDJ = JB + 4;
constexpr float kRange = 60.f;  // largest |g - g_m| (nats) of the fp32 factorised decays

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

__device__ __forceinline__ float ld_act(const void* p, int64_t i, bool bf16) {
  return bf16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(p)[i]) : static_cast<const float*>(p)[i];
}

__device__ __forceinline__ void cp_async16(float* dst, const float* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" :: "r"((uint32_t)__cvta_generic_to_shared(dst)),
               "l"(src) : "memory");
}
// 16-byte cp.async reading 16 bytes (valid) or none (zero fill)
__device__ __forceinline__ void cp_async16z(float* dst, const float* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" :: "r"((uint32_t)__cvta_generic_to_shared(dst)),
               "l"(src), "r"(valid ? 16u : 0u) : "memory");
}
__device__ __forceinline__ void cp_async16v(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" :: "r"((uint32_t)__cvta_generic_to_shared(dst)),
               "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// Per chunk-head arrays in the workspace, fp32, chunk-head index (b * H + h) * nc + c.
struct CbwdBufs {
  float* W;    // [CH][D]  T KG
  float* Ut;   // [CH][D]  T V
  float* Kt;   // [CH][D]  k e^{gl - g}
  float* Z;    // [CH][D]  P^T dO
  float* Y;    // [D][D]   QG^T dO
  float* X;    // [CH][CH] (I + A)^{-1}
  float* Ab;   // [CH][CH] A / beta_r
  float* egl;  // [D]      e^{gl}
  float* S;    // [D][D]   state entering the chunk
  float* U;    // [CH][D]  U~ - W S
  float* dS;   // [D][D]   gradient reaching the chunk's exit state
  float* dU;   // [CH][D]
  float* dQG;  // [CH][D]  dO S^T
  float* dW;   // [CH][D]  -dU S^T
  float* dKt;  // [CH][D]  U dS^T
  float* dP;   // [CH][CH] lower(dO U^T)
  float* dUV;  // [CH][CH] dU V^T
  float* last; // [D]      e^{gl} rowsum(dS o S)
};

struct CbwdArgs {
  const float* q; const float* k; const float* v;   // convolved activations, fp32 [B][N][H][D]
  const float* la;                                   // [B][N][H][D]
  const void* beta;                                  // [B][N][H], dtype
  const void* d_o;                                   // [B][N][H][D], dtype
  const float* S0;                                   // [B][H][D][D] or null
  const float* dSN;                                  // [B][H][D][D] or null
  float* dq; float* dk; float* dv;                   // fp32 [B][N][H][D]
  float* dla;                                        // fp32 [B][N][H][D]
  float* dbeta;                                      // fp32 [B][N][H]
  float* dS0;                                        // [B][H][D][D] or null
  CbwdBufs w;
  int64_t N; int H; int nc; bool bf16;
  uint32_t* status;
};

// ---- warp-level tensor-core products (mma.sync m16n8k8, tf32) ----------------------
// Each operand is split as x = hi + lo (both tf32) and a product is formed as
// hi*hi + hi*lo + lo*hi, which keeps it at about fp32 accuracy (relative error near 2^-20).
__device__ __forceinline__ void split_tf32(float x, uint32_t& hi, uint32_t& lo) {
  // hi: x with the 13 low mantissa bits cleared (a tf32 value); lo: the exact remainder x - hi,
  // cleared the same way (its dropped bits are below 2^-20 of |x|)
  hi = __float_as_uint(x) & 0xffffe000u;
  lo = __float_as_uint(x - __uint_as_float(hi)) & 0xffffe000u;
}
__device__ __forceinline__ uint32_t tf32_rn(float x) {   // nearest tf32 (single-product mode)
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
  asm volatile("mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
               : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
               : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// One warp: c[mt][nt] += the 16 x 8 tile (rows m0 + 16 mt, columns n0 + 8 nt) of A B, K a
// multiple of 8, A(m, k) = A[m * am + k * ak] and B(k, n) = B[k * bk + n * bn] in shared memory.
// Fragment coordinates, g = lane / 4, t = lane % 4: c[.][.][0..3] = C[g][2t], C[g][2t+1],
// C[g+8][2t], C[g+8][2t+1] of the tile.  With CHAINS the hi*hi and the correction products of
// even and odd k-steps go to four separate accumulators (summed at the end), for warps that
// own one or two tiles and would otherwise wait on each product.  Shared-memory reads are free
// of bank conflicts when a row stride along k (am or bn = ld, the other 1) is 4 mod 32 and a
// row stride across k (ak or bk = ld) is 8 mod 32.  SPLIT = false forms one product of the
// operands rounded to the nearest tf32 (relative error near 2^-11, as an fp16 operand).
template <int MT, int NT, bool CHAINS = false, bool SPLIT = true>
__device__ __forceinline__ void wmma3(float (&c)[MT][NT][4], const float* A, int am, int ak, const float* B, int bk,
                                      int bn, int K, int m0, int n0, int lane) {
  if (!SPLIT) {
    const int g = lane >> 2, t = lane & 3;
    const float* a0 = A + (m0 + g) * am + t * ak;
    const float* b0 = B + t * bk + (n0 + g) * bn;
#pragma unroll 2
    for (int k0 = 0; k0 < K; k0 += 8) {
      uint32_t ah[MT][4], bh[NT][2];
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        const float* p = a0 + 16 * mt * am + k0 * ak;
        ah[mt][0] = tf32_rn(p[0]);
        ah[mt][1] = tf32_rn(p[8 * am]);
        ah[mt][2] = tf32_rn(p[4 * ak]);
        ah[mt][3] = tf32_rn(p[8 * am + 4 * ak]);
      }
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const float* p = b0 + k0 * bk + 8 * nt * bn;
        bh[nt][0] = tf32_rn(p[0]);
        bh[nt][1] = tf32_rn(p[4 * bk]);
      }
#pragma unroll
      for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma_tf32(c[mt][nt], ah[mt], bh[nt]);
    }
    return;
  }
  const int g = lane >> 2, t = lane & 3;
  const float* a0 = A + (m0 + g) * am + t * ak;
  const float* b0 = B + t * bk + (n0 + g) * bn;
  float e[CHAINS ? 3 : 1][MT][NT][4];
  if (CHAINS) {
#pragma unroll
    for (int x = 0; x < (CHAINS ? 3 : 1); ++x)
#pragma unroll
      for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int i = 0; i < 4; ++i) e[x][mt][nt][i] = 0.f;
  }
#pragma unroll 2
  for (int k0 = 0; k0 < K; k0 += 8) {
    uint32_t ah[MT][4], al[MT][4], bh[NT][2], bl[NT][2];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      const float* p = a0 + 16 * mt * am + k0 * ak;
      split_tf32(p[0], ah[mt][0], al[mt][0]);
      split_tf32(p[8 * am], ah[mt][1], al[mt][1]);
      split_tf32(p[4 * ak], ah[mt][2], al[mt][2]);
      split_tf32(p[8 * am + 4 * ak], ah[mt][3], al[mt][3]);
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const float* p = b0 + k0 * bk + 8 * nt * bn;
      split_tf32(p[0], bh[nt][0], bl[nt][0]);
      split_tf32(p[4 * bk], bh[nt][1], bl[nt][1]);
    }
    const bool odd = CHAINS && ((k0 >> 3) & 1);
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        if (CHAINS) {
          mma_tf32(e[odd ? 1 : 0][mt][nt], al[mt], bh[nt]);
          mma_tf32(e[odd ? 1 : 0][mt][nt], ah[mt], bl[nt]);
          if (odd) mma_tf32(e[2][mt][nt], ah[mt], bh[nt]);
          else mma_tf32(c[mt][nt], ah[mt], bh[nt]);
        } else {
          mma_tf32(c[mt][nt], al[mt], bh[nt]);
          mma_tf32(c[mt][nt], ah[mt], bl[nt]);
          mma_tf32(c[mt][nt], ah[mt], bh[nt]);
        }
      }
  }
  if (CHAINS) {
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) c[mt][nt][i] += (e[0][mt][nt][i] + e[1][mt][nt][i]) + e[2][mt][nt][i];
  }
}

template <int MT, int NT>
__device__ __forceinline__ void zero4(float (&c)[MT][NT][4]) {
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) c[mt][nt][i] = 0.f;
}

// rows [0, CH) of a [.][W] fp32 matrix whose row r starts at src + r * rs into shared memory
// (row stride ld) by cp.async, zero from row n on; the caller commits and waits
template <int W>
__device__ __forceinline__ void stage_rows(float* dst, int ld, const float* src, int64_t rs, int n, int tid) {
  for (int idx = tid; idx < CH * W / 4; idx += NT) {
    const int r = idx / (W / 4), c4 = (idx % (W / 4)) * 4;
    cp_async16z(dst + r * ld + c4, r < n ? src + r * rs + c4 : src, r < n);
  }
}

// 8 consecutive activations of dtype (bf16 or fp32) from element i (a multiple of 8), as floats
__device__ __forceinline__ void ld8_act(const void* p, int64_t i, bool bf16, float (&v)[8]) {
  if (bf16) {
    const uint4 u = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p) + i);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      v[2 * j] = __uint_as_float(w[j] << 16);
      v[2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
    }
  } else {
    const float4 x0 = *reinterpret_cast<const float4*>(static_cast<const float*>(p) + i);
    const float4 x1 = *reinterpret_cast<const float4*>(static_cast<const float*>(p) + i + 4);
    v[0] = x0.x; v[1] = x0.y; v[2] = x0.z; v[3] = x0.w;
    v[4] = x1.x; v[5] = x1.y; v[6] = x1.z; v[7] = x1.w;
  }
}

// running sum over the chunk's rows, per key channel (threads < D); per channel g_m, g_l,
// e^{g_m} and e^{g_l - g_m}
template <int D>
__device__ __forceinline__ void chunk_cumsum(float* Gs, float* gm, float* gl, float* egm, float* eglm, int tid) {
  constexpr int LDD = D + 4;
  if (tid < D) {
    float s = 0.f, m = 0.f;
    for (int r = 0; r < CH; ++r) {
      s += Gs[r * LDD + tid];
      Gs[r * LDD + tid] = s;
      if (r == CH / 2 - 1) m = s;
    }
    gm[tid] = m;
    gl[tid] = s;
    egm[tid] = expf(m);
    eglm[tid] = expf(s - m);
  }
}

struct ChunkPos {
  int64_t ch;     // chunk-head index
  int64_t tok0;   // (b * N + n0) * H + h: token row index of the chunk's first token
  int n;          // tokens in the chunk
};

__device__ __forceinline__ ChunkPos chunk_pos(const CbwdArgs& a) {
  const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int64_t n0 = (int64_t)c * CH;
  ChunkPos p;
  p.ch = ((int64_t)b * a.H + h) * a.nc + c;
  p.tok0 = ((int64_t)b * a.N + n0) * a.H + h;
  p.n = (int)(a.N - n0 < CH ? a.N - n0 : CH);
  return p;
}

// ---- per-chunk forward quantities and dO terms ------------------------------------
// Warp tilings of the per-chunk products (8 warps, wmma3 tiles of 16 x 8):
//   CH x CH: warp block 16 x 32 at (16 (w % 4), 32 (w / 4))
//   CH x D:  warp block 32 x D/4 at (32 (w % 2), D/4 (w / 2))
//   D x D:   warp block D/4 x D/2 at (D/4 (w % 4), D/2 (w / 4))
// A thread's elements of a block: rows m0 + 16 mt + g (+ 8), columns n0 + 8 nt + 2t (+ 1).
#define FRAG_LOOP(MT, NT_)                    \
  _Pragma("unroll") for (int mt = 0; mt < (MT); ++mt) \
  _Pragma("unroll") for (int nt = 0; nt < (NT_); ++nt) \
  _Pragma("unroll") for (int i = 0; i < 4; ++i)
#define FRAG_R(m0) ((m0) + 16 * mt + g + 8 * (i >> 1))
#define FRAG_C(n0) ((n0) + 8 * nt + 2 * t + (i & 1))

// A warp's accumulator tiles into a row-major [.][ld] array at element offset off: fp32, or, for
// bf16 problems (!SPLIT), fp16 at the same element offset (what the chains read: W and their
// additive terms)
template <int MT, int NT_, bool SPLIT>
__device__ __forceinline__ void store_tile(float* base, int64_t off, int ld, const float (&acc)[MT][NT_][4], int m0,
                                           int n0, int g, int t) {
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int nt = 0; nt < NT_; ++nt)
#pragma unroll
      for (int hi = 0; hi < 2; ++hi) {
        const int r = m0 + 16 * mt + g + 8 * hi, c = n0 + 8 * nt + 2 * t;
        if (SPLIT) {
          *reinterpret_cast<float2*>(base + off + r * ld + c) = make_float2(acc[mt][nt][2 * hi], acc[mt][nt][2 * hi + 1]);
        } else {
          *reinterpret_cast<__half2*>(reinterpret_cast<__half*>(base) + off + r * ld + c) =
              __floats2half2_rn(acc[mt][nt][2 * hi], acc[mt][nt][2 * hi + 1]);
        }
      }
}

template <int D>
constexpr size_t prep_smem() { return sizeof(float) * (4 * CH * (D + 4) + 2 * CH * LDC + 4 * D + CH); }

template <int D, bool SPLIT>
__global__ void __launch_bounds__(NT, 1) cbwd_prep_kernel(CbwdArgs a) {
  constexpr int LDD = D + 4, NTD = D / 32;
  extern __shared__ __align__(16) float sm[];
  float* Gs = sm;                 // [CH][LDD] g, later dO
  float* Kx = Gs + CH * LDD;      // k e^{g - g_m}
  float* KN = Kx + CH * LDD;      // k e^{g_m - g}, later v
  float* Qx = KN + CH * LDD;      // q e^{g - g_m}
  float* As = Qx + CH * LDD;      // [CH][LDC] A, later T
  float* Ps = As + CH * LDC;      // P
  float* gm = Ps + CH * LDC;      // [D]
  float* gl = gm + D;             // [D]
  float* egm = gl + D;            // [D] e^{g_m}
  float* eglm = egm + D;          // [D] e^{g_l - g_m}
  float* bs = eglm + D;           // [CH] beta
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, g = lane >> 2, t = lane & 3;
  const ChunkPos p = chunk_pos(a);
  const int64_t rs = (int64_t)a.H * D;
  // log alpha, k and q of the chunk in flight together (k and q land raw in Kx and Qx)
  stage_rows<D>(Gs, LDD, a.la + p.tok0 * D, rs, p.n, tid);
  stage_rows<D>(Kx, LDD, a.k + p.tok0 * D, rs, p.n, tid);
  stage_rows<D>(Qx, LDD, a.q + p.tok0 * D, rs, p.n, tid);
  cp_async_commit();
  if (tid < CH) bs[tid] = tid < p.n ? ld_act(a.beta, p.tok0 + (int64_t)tid * a.H, a.bf16) : 0.f;
  cp_async_wait_all();
  __syncthreads();
  chunk_cumsum<D>(Gs, gm, gl, egm, eglm, tid);
  __syncthreads();
  bool bad = false;
  float* Kt = a.w.Kt + p.ch * CH * D;
  __half* Kth = reinterpret_cast<__half*>(a.w.Kt) + p.ch * CH * D;
  for (int idx = tid; idx < CH * D / 4; idx += NT) {   // each thread transforms its own elements in place
    const int r = idx / (D / 4), c4 = (idx % (D / 4)) * 4;
    const float4 k4 = *reinterpret_cast<const float4*>(Kx + r * LDD + c4);
    const float4 q4 = *reinterpret_cast<const float4*>(Qx + r * LDD + c4);
    const float4 g4 = *reinterpret_cast<const float4*>(Gs + r * LDD + c4);
    const float kv[4] = {k4.x, k4.y, k4.z, k4.w}, qv[4] = {q4.x, q4.y, q4.z, q4.w}, gv[4] = {g4.x, g4.y, g4.z, g4.w};
    float kx[4], kn[4], qx[4], kt[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float x = gv[j] - gm[c4 + j];
      bad |= fabsf(x) > kRange;
      const float ep = expf(x), en = __fdividef(1.f, ep);   // |x| <= kRange: both well inside fp32
      kx[j] = kv[j] * ep;
      kn[j] = kv[j] * en;
      qx[j] = qv[j] * ep;
      kt[j] = kv[j] * (eglm[c4 + j] * en);                  // e^{g_l - g}
    }
    *reinterpret_cast<float4*>(Kx + r * LDD + c4) = make_float4(kx[0], kx[1], kx[2], kx[3]);
    *reinterpret_cast<float4*>(KN + r * LDD + c4) = make_float4(kn[0], kn[1], kn[2], kn[3]);
    *reinterpret_cast<float4*>(Qx + r * LDD + c4) = make_float4(qx[0], qx[1], qx[2], qx[3]);
    if (SPLIT) {
      *reinterpret_cast<float4*>(Kt + r * D + c4) = make_float4(kt[0], kt[1], kt[2], kt[3]);
    } else {   // fp16 operand of the chains
      const __half2 h0 = __floats2half2_rn(kt[0], kt[1]), h1 = __floats2half2_rn(kt[2], kt[3]);
      *reinterpret_cast<uint2*>(Kth + r * D + c4) =
          make_uint2(*reinterpret_cast<const uint32_t*>(&h0), *reinterpret_cast<const uint32_t*>(&h1));
    }
  }
  if (tid < D) a.w.egl[p.ch * D + tid] = expf(gl[tid]);
  if (__syncthreads_or(bad) && tid == 0) set_status(a.status, KDA_ERR_RANGE);

  {  // A = Diag(beta) strict(Kx KN^T), P = lower(Qx KN^T)
    const int m0 = 16 * (warp & 3), n0 = 32 * (warp >> 2);
    float ab[1][4][4], pp[1][4][4];
    zero4(ab);
    zero4(pp);
    wmma3<1, 4, false, SPLIT>(ab, Kx, LDD, 1, KN, 1, LDD, D, m0, n0, lane);
    wmma3<1, 4, false, SPLIT>(pp, Qx, LDD, 1, KN, 1, LDD, D, m0, n0, lane);
    float* Abg = a.w.Ab + p.ch * CH * CH;
    FRAG_LOOP(1, 4) {
      const int r = FRAG_R(m0), c = FRAG_C(n0);
      const float abv = c < r ? ab[mt][nt][i] : 0.f;
      As[r * LDC + c] = bs[r] * abv;
      Abg[r * CH + c] = abv;
      Ps[r * LDC + c] = c <= r ? pp[mt][nt][i] : 0.f;
    }
  }
  __syncthreads();
  // v into the KN tile the products above no longer read, by cp.async
  stage_rows<D>(KN, LDD, a.v + p.tok0 * D, rs, p.n, tid);
  cp_async_commit();
  // X = (I + A)^{-1} by forward substitution, one column per thread (threads < CH); the other
  // threads meanwhile convert dO into the g tile
  float x[CH];
  if (tid < CH) {
#pragma unroll
    for (int r = 0; r < CH; ++r) {
      float s0 = r == tid ? 1.f : 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
      for (int i = 0; i + 3 < r; i += 4) {
        const float4 a4 = *reinterpret_cast<const float4*>(As + r * LDC + i);
        s0 = fmaf(-a4.x, x[i], s0);
        s1 = fmaf(-a4.y, x[i + 1], s1);
        s2 = fmaf(-a4.z, x[i + 2], s2);
        s3 = fmaf(-a4.w, x[i + 3], s3);
      }
#pragma unroll
      for (int i = r & ~3; i < r; ++i) s0 = fmaf(-As[r * LDC + i], x[i], s0);
      x[r] = (s0 + s1) + (s2 + s3);
    }
    float* Xg = a.w.X + p.ch * CH * CH;
#pragma unroll
    for (int r = 0; r < CH; ++r) Xg[r * CH + tid] = x[r];
  } else {
    constexpr int N8 = CH * D / 8, PER = (N8 + NT - CH - 1) / (NT - CH);
    float v8[PER][8];
#pragma unroll
    for (int it = 0; it < PER; ++it) {   // all loads first, then the stores
      const int idx = tid - CH + it * (NT - CH), r = idx / (D / 8), c8 = (idx % (D / 8)) * 8;
      if (idx < N8 && r < p.n) ld8_act(a.d_o, (p.tok0 + (int64_t)r * a.H) * D + c8, a.bf16, v8[it]);
      else
#pragma unroll
        for (int j = 0; j < 8; ++j) v8[it][j] = 0.f;
    }
#pragma unroll
    for (int it = 0; it < PER; ++it) {
      const int idx = tid - CH + it * (NT - CH), r = idx / (D / 8), c8 = (idx % (D / 8)) * 8;
      if (idx < N8) {
        *reinterpret_cast<float4*>(Gs + r * LDD + c8) = make_float4(v8[it][0], v8[it][1], v8[it][2], v8[it][3]);
        *reinterpret_cast<float4*>(Gs + r * LDD + c8 + 4) = make_float4(v8[it][4], v8[it][5], v8[it][6], v8[it][7]);
      }
    }
  }
  cp_async_wait_all();
  __syncthreads();
  if (tid < CH) {
#pragma unroll
    for (int r = 0; r < CH; ++r) As[r * LDC + tid] = x[r] * bs[tid];   // T = X Diag(beta)
  }
  __syncthreads();
  {  // W = T Kx Diag(e^{g_m}),  U~ = T V,  Z = P^T dO
    const int m0 = 32 * (warp & 1), n0 = (D / 4) * (warp >> 1);
    float acc[2][NTD][4];
    zero4(acc);
    wmma3<2, NTD, false, SPLIT>(acc, As, LDC, 1, Kx, LDD, 1, CH, m0, n0, lane);
    FRAG_LOOP(2, NTD) acc[mt][nt][i] *= egm[FRAG_C(n0)];
    store_tile<2, NTD, SPLIT>(a.w.W, p.ch * CH * D, D, acc, m0, n0, g, t);
    zero4(acc);
    wmma3<2, NTD, false, SPLIT>(acc, As, LDC, 1, KN, LDD, 1, CH, m0, n0, lane);
    store_tile<2, NTD, SPLIT>(a.w.Ut, p.ch * CH * D, D, acc, m0, n0, g, t);
    zero4(acc);
    wmma3<2, NTD, false, SPLIT>(acc, Ps, 1, LDC, Gs, LDD, 1, CH, m0, n0, lane);
    store_tile<2, NTD, SPLIT>(a.w.Z, p.ch * CH * D, D, acc, m0, n0, g, t);
  }
  {  // Y = QG^T dO = Diag(e^{g_m}) Qx^T dO
    const int m0 = (D / 4) * (warp & 3), n0 = (D / 2) * (warp >> 2);
    float acc[D / 64][D / 16][4];
    zero4(acc);
    wmma3<D / 64, D / 16, false, SPLIT>(acc, Qx, 1, LDD, Gs, LDD, 1, CH, m0, n0, lane);
    FRAG_LOOP(D / 64, D / 16) acc[mt][nt][i] *= egm[FRAG_R(m0)];
    store_tile<D / 64, D / 16, SPLIT>(a.w.Y, p.ch * D * D, D, acc, m0, n0, g, t);
  }
}

// ---- the two serial passes over chunks, CW value columns per CTA ------------------------
// Column j of the state (and of its gradient) only meets column j of v and dO, so the
// (b, h) chains split into D / CW independent CTAs.  The next chunk's tiles are copied by
// cp.async into the other half of a double buffer while the current chunk is processed.
// Tile strides: the tile read along k by the first product (W forward, Kt backward) is
// D + 4 wide, the one read across k by the second (Kt forward, W backward) D + 8, the
// state and U columns CW + 8 (see wmma3).
template <int D>
struct ChainLd {
  static constexpr int L1 = D + 4, L2 = D + 8, LS = CW + 8;
};

template <int D, bool BWD>
constexpr size_t chain_smem() {
  using L = ChainLd<D>;
  return sizeof(float) * (2 * CH * (L::L1 + L::L2) + 2 * CH * CW + (BWD ? 2 * D * CW : 0) + 2 * D + D * L::LS +
                          CH * L::LS);
}

template <int D, bool BWD>
__global__ void __launch_bounds__(NT, 1) cbwd_chain_kernel(CbwdArgs a) {
  using L = ChainLd<D>;
  constexpr int LS = L::LS;
  extern __shared__ __align__(16) float sm[];
  float* T1 = sm;                            // [2][CH][L1]  W (forward) or Kt (backward): first product
  float* T2 = T1 + 2 * CH * L::L1;           // [2][CH][L2]  Kt (forward) or W (backward): second product
  float* Vb = T2 + 2 * CH * L::L2;           // [2][CH][CW]  U~ (forward) or Z (backward) columns
  float* Yb = Vb + 2 * CH * CW;              // [2][D][CW]   Y columns (backward)
  float* eb = Yb + (BWD ? 2 * D * CW : 0);   // [2][D]       e^{gl}
  float* S = eb + 2 * D;                     // [D][LS]      state (forward) or its gradient (backward)
  float* Us = S + D * LS;                    // [CH][LS]     U or dU
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c0 = blockIdx.x * CW, h = blockIdx.y, b = blockIdx.z;
  const int64_t bh = (int64_t)b * a.H + h, ch0 = bh * a.nc;
  const float* init = BWD ? a.dSN : a.S0;
  for (int idx = tid; idx < D * CW; idx += NT) {
    const int r = idx / CW, j = idx % CW;
    S[r * LS + j] = init ? init[(bh * D + r) * D + c0 + j] : 0.f;
  }
  auto issue = [&](int c) {
    if (c >= 0 && c < a.nc) {
      const int s = c & 1;
      const int64_t ch = ch0 + c;
      const float* M1 = (BWD ? a.w.Kt : a.w.W) + ch * CH * D;
      const float* M2 = (BWD ? a.w.W : a.w.Kt) + ch * CH * D;
      const float* V = (BWD ? a.w.Z : a.w.Ut) + ch * CH * D;
      for (int i = tid; i < CH * D / 4; i += NT) {
        const int r = i / (D / 4), c4 = (i % (D / 4)) * 4;
        cp_async16(T1 + (s * CH + r) * L::L1 + c4, M1 + r * D + c4);
        cp_async16(T2 + (s * CH + r) * L::L2 + c4, M2 + r * D + c4);
      }
      for (int i = tid; i < CH * CW / 4; i += NT) {
        const int r = i / (CW / 4), c4 = (i % (CW / 4)) * 4;
        cp_async16(Vb + (s * CH + r) * CW + c4, V + r * D + c0 + c4);
      }
      if (BWD) {
        const float* Y = a.w.Y + ch * D * D;
        for (int i = tid; i < D * CW / 4; i += NT) {
          const int r = i / (CW / 4), c4 = (i % (CW / 4)) * 4;
          cp_async16(Yb + (s * D + r) * CW + c4, Y + r * D + c0 + c4);
        }
      }
      for (int i = tid; i < D / 4; i += NT) cp_async16(eb + s * D + 4 * i, a.w.egl + ch * D + 4 * i);
    }
    cp_async_commit();
  };
  // warp tiles: the CH x CW product as 4 x 2 tiles of 16 x 8, one per warp; the D x CW product
  // as (D / 16) x 2 tiles, D / 64 per warp
  const int g = lane >> 2, t = lane & 3;
  const int m1 = 16 * (warp & 3), n1 = 8 * (warp >> 2);
  constexpr int MT2 = D / 64;
  const int m2 = 16 * MT2 * (warp & 3), n2 = 8 * (warp >> 2);
  issue(BWD ? a.nc - 1 : 0);
  for (int step = 0; step < a.nc; ++step) {
    const int c = BWD ? a.nc - 1 - step : step;
    const int s = c & 1;
    const int64_t ch = ch0 + c;
    cp_async_wait_all();
    __syncthreads();   // chunk c's tiles in place; every thread is done with the other buffer
    issue(BWD ? c - 1 : c + 1);
    {  // the state entering the chunk (forward) or the gradient reaching its exit (backward)
      float* out = (BWD ? a.w.dS : a.w.S) + ch * D * D;
      for (int idx = tid; idx < D * CW; idx += NT) {
        const int r = idx / CW, j = idx % CW;
        out[r * D + c0 + j] = S[r * LS + j];
      }
    }
    {  // forward: U = U~ - W S;  backward: dU = Z + Kt dS
      float u[1][1][4];
      zero4(u);
      wmma3<1, 1, true>(u, T1 + s * CH * L::L1, L::L1, 1, S, LS, 1, D, m1, n1, lane);
      float* out = (BWD ? a.w.dU : a.w.U) + ch * CH * D;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = m1 + g + 8 * (i >> 1), j = n1 + 2 * t + (i & 1);
        const float val = BWD ? Vb[(s * CH + r) * CW + j] + u[0][0][i] : Vb[(s * CH + r) * CW + j] - u[0][0][i];
        Us[r * LS + j] = val;
        out[r * D + c0 + j] = val;
      }
    }
    __syncthreads();
    {  // forward: S = Diag(e^{gl}) S + Kt^T U;  backward: dS = Diag(e^{gl}) dS - W^T dU + Y
      float sv[MT2][1][4];
      zero4(sv);
      wmma3<MT2, 1, true>(sv, T2 + s * CH * L::L2, 1, L::L2, Us, LS, 1, CH, m2, n2, lane);
#pragma unroll
      for (int mt = 0; mt < MT2; ++mt)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int r = m2 + 16 * mt + g + 8 * (i >> 1), j = n2 + 2 * t + (i & 1);
          const float prev = eb[s * D + r] * S[r * LS + j];
          S[r * LS + j] = BWD ? prev - sv[mt][0][i] + Yb[(s * D + r) * CW + j] : prev + sv[mt][0][i];
        }
    }
  }
  if (BWD && a.dS0) {
    __syncthreads();
    for (int idx = tid; idx < D * CW; idx += NT) {
      const int r = idx / CW, j = idx % CW;
      a.dS0[(bh * D + r) * D + c0 + j] = S[r * LS + j];
    }
  }
}

// ---- the two chains of bf16 problems: fp16 operands, one launch ---------------------------
// W and Kt arrive in fp16 (written so by the prep kernel), and the state (or its gradient) and U
// (or dU) enter the products as fp16 images, which accumulate in fp32 on mma.sync m16n8k16: the
// operand precision of the forward's tensor-core state pass.  The state itself stays fp32 in
// shared memory; each update also writes its fp16 image, transposed (value column major) so that
// the B fragments of both products load by ldmatrix, like the A fragments.  The forward chain (S
// of every chunk) and the reverse chain (dS) do not depend on each other, so both run in one
// launch, blockIdx.z = 2 b + direction, two CTAs per SM.  Row strides: the fp16 tiles and images
// a multiple of 16 bytes and 4 mod 32 words (ldmatrix free of bank conflicts); the fp32 state CW + 8
// (the update's 8-byte accesses free of bank conflicts).
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void mma_f16(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
  asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
               : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
               : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}
template <int D>
struct ChainH {
  static constexpr int LH = D + 8;    // W / Kt tiles, halves per row
  static constexpr int LT = D + 8;    // fp16 image of the state, [CW][LT]: value column major
  static constexpr int LU = CH + 8;   // fp16 image of U, [CW][LU]
  static constexpr int LS = CW + 8;   // fp32 state, [D][LS]
};

template <int D>
constexpr size_t chain_h_smem() {
  using L = ChainH<D>;
  return sizeof(__half) * (2 * 2 * CH * L::LH + CW * L::LT + CW * L::LU + 2 * CH * CW + 2 * D * CW) +
         sizeof(float) * (2 * D + D * L::LS);
}

template <int D, bool BWD>
__device__ __forceinline__ void chain_h_pass(const CbwdArgs& a, int b, uint8_t* smraw) {
  using L = ChainH<D>;
  constexpr int LH = L::LH, LT = L::LT, LU = L::LU, LS = L::LS;
  __half* T1 = reinterpret_cast<__half*>(smraw);           // [2][CH][LH] W (forward) or Kt (backward)
  __half* T2 = T1 + 2 * CH * LH;                            // [2][CH][LH] Kt (forward) or W (backward)
  __half* ST = T2 + 2 * CH * LH;                            // [CW][LT]    fp16 state, transposed
  __half* UT = ST + CW * LT;                                // [CW][LU]    fp16 U or dU, transposed
  __half* Vb = UT + CW * LU;                                // [2][CH][CW] U~ (forward) or Z (backward), fp16
  __half* Yb = Vb + 2 * CH * CW;                            // [2][D][CW]  Y columns (backward), fp16
  float* eb = reinterpret_cast<float*>(Yb + 2 * D * CW);    // [2][D]      e^{gl}
  float* S = eb + 2 * D;                                    // [D][LS]     state or its gradient
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c0 = blockIdx.x * CW, h = blockIdx.y;
  const int64_t bh = (int64_t)b * a.H + h, ch0 = bh * a.nc;
  const float* init = BWD ? a.dSN : a.S0;
  for (int idx = tid; idx < D * CW; idx += NT) {
    const int r = idx / CW, j = idx % CW;
    const float v = init ? init[(bh * D + r) * D + c0 + j] : 0.f;
    S[r * LS + j] = v;
    ST[j * LT + r] = __float2half_rn(v);
  }
  const __half* H1 = reinterpret_cast<const __half*>(BWD ? a.w.Kt : a.w.W);
  const __half* H2 = reinterpret_cast<const __half*>(BWD ? a.w.W : a.w.Kt);
  auto issue = [&](int c) {
    if (c >= 0 && c < a.nc) {
      const int s = c & 1;
      const int64_t ch = ch0 + c;
      const __half* M1 = H1 + ch * CH * D;
      const __half* M2 = H2 + ch * CH * D;
      const __half* V = reinterpret_cast<const __half*>(BWD ? a.w.Z : a.w.Ut) + ch * CH * D;
      for (int i = tid; i < CH * D / 8; i += NT) {
        const int r = i / (D / 8), c8 = (i % (D / 8)) * 8;
        cp_async16v(T1 + (s * CH + r) * LH + c8, M1 + r * D + c8);
        cp_async16v(T2 + (s * CH + r) * LH + c8, M2 + r * D + c8);
      }
      for (int i = tid; i < CH * CW / 8; i += NT) {
        const int r = i / (CW / 8), c8 = (i % (CW / 8)) * 8;
        cp_async16v(Vb + (s * CH + r) * CW + c8, V + r * D + c0 + c8);
      }
      if (BWD) {
        const __half* Y = reinterpret_cast<const __half*>(a.w.Y) + ch * D * D;
        for (int i = tid; i < D * CW / 8; i += NT) {
          const int r = i / (CW / 8), c8 = (i % (CW / 8)) * 8;
          cp_async16v(Yb + (s * D + r) * CW + c8, Y + r * D + c0 + c8);
        }
      }
      for (int i = tid; i < D / 4; i += NT) cp_async16(eb + s * D + 4 * i, a.w.egl + ch * D + 4 * i);
    }
    cp_async_commit();
  };
  // warp tiles: the CH x CW product as 4 x 2 tiles of 16 x 8, one per warp; the D x CW product
  // as (D / 16) x 2 tiles, D / 64 per warp
  const int g = lane >> 2, t = lane & 3;
  const int m1 = 16 * (warp & 3), n1 = 8 * (warp >> 2);
  constexpr int MT2 = D / 64;
  const int m2 = 16 * MT2 * (warp & 3), n2 = 8 * (warp >> 2);
  // ldmatrix row addresses.  A of a row-major tile (rows m, 16-half steps along k): matrices
  // (m 0-7, k 0-7), (m 8-15, k 0-7), (m 0-7, k 8-15), (m 8-15, k 8-15).  A of a tile stored
  // transposed (rows k): the same four, read with .trans.  B from a value-column-major image
  // (rows n): matrices k 0-7, 8-15, 16-23, 24-31, i.e. the B fragments of two k-steps.
  const int ar = (lane & 7) + 8 * ((lane >> 3) & 1), ac = 8 * (lane >> 4);
  const int tr = (lane & 7) + 8 * (lane >> 4), tc = 8 * ((lane >> 3) & 1);
  const int br = lane & 7, bc = 8 * (lane >> 3);
  const uint32_t t1_0 = (uint32_t)__cvta_generic_to_shared(T1 + (m1 + ar) * LH + ac);
  const uint32_t t2_0 = (uint32_t)__cvta_generic_to_shared(T2 + tr * LH + m2 + tc);
  const uint32_t st_0 = (uint32_t)__cvta_generic_to_shared(ST + (n1 + br) * LT + bc);
  const uint32_t ut_0 = (uint32_t)__cvta_generic_to_shared(UT + (n2 + br) * LU + bc);
  issue(BWD ? a.nc - 1 : 0);
  for (int step = 0; step < a.nc; ++step) {
    const int c = BWD ? a.nc - 1 - step : step;
    const int s = c & 1;
    const int64_t ch = ch0 + c;
    cp_async_wait_all();
    __syncthreads();   // chunk c's tiles in place, the state and its image updated; every thread is
                       // done with the other buffer
    issue(BWD ? c - 1 : c + 1);
    {  // the state entering the chunk (forward) or the gradient reaching its exit (backward)
      float* out = (BWD ? a.w.dS : a.w.S) + ch * D * D;
#pragma unroll
      for (int i = 0; i < D * CW / 4 / NT; ++i) {
        const int idx = tid + i * NT, r = idx / (CW / 4), j4 = (idx % (CW / 4)) * 4;
        *reinterpret_cast<float4*>(out + r * D + c0 + j4) = *reinterpret_cast<const float4*>(S + r * LS + j4);
      }
    }
    {  // forward: U = U~ - W S;  backward: dU = Z + Kt dS
      float u[4] = {0.f, 0.f, 0.f, 0.f}, u2[4] = {0.f, 0.f, 0.f, 0.f};
      const uint32_t abase = t1_0 + (uint32_t)(s * CH * LH * 2);
#pragma unroll
      for (int k2 = 0; k2 < D / 32; ++k2) {
        uint32_t bq[4], af[4];
        ldsm_x4(bq, st_0 + 64u * k2);
        ldsm_x4(af, abase + 64u * k2);
        mma_f16(u, af, {bq[0], bq[1]});
        ldsm_x4(af, abase + 64u * k2 + 32u);
        mma_f16(u2, af, {bq[2], bq[3]});
      }
      float* out = (BWD ? a.w.dU : a.w.U) + ch * CH * D;
#pragma unroll
      for (int hi = 0; hi < 2; ++hi) {
        const int r = m1 + g + 8 * hi, j = n1 + 2 * t;
        const float2 vb = __half22float2(*reinterpret_cast<const __half2*>(Vb + (s * CH + r) * CW + j));
        const float p0 = u[2 * hi] + u2[2 * hi], p1 = u[2 * hi + 1] + u2[2 * hi + 1];
        const float v0 = BWD ? vb.x + p0 : vb.x - p0, v1 = BWD ? vb.y + p1 : vb.y - p1;
        UT[j * LU + r] = __float2half_rn(v0);
        UT[(j + 1) * LU + r] = __float2half_rn(v1);
        *reinterpret_cast<float2*>(out + r * D + c0 + j) = make_float2(v0, v1);
      }
    }
    __syncthreads();
    {  // forward: S = Diag(e^{gl}) S + Kt^T U;  backward: dS = Diag(e^{gl}) dS - W^T dU + Y
      float sv[MT2][4];
#pragma unroll
      for (int mt = 0; mt < MT2; ++mt)
#pragma unroll
        for (int i = 0; i < 4; ++i) sv[mt][i] = 0.f;
      const uint32_t abase = t2_0 + (uint32_t)(s * CH * LH * 2);
#pragma unroll
      for (int k2 = 0; k2 < CH / 32; ++k2) {
        uint32_t bq[4];
        ldsm_x4(bq, ut_0 + 64u * k2);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const int kk = 2 * k2 + half;
#pragma unroll
          for (int mt = 0; mt < MT2; ++mt) {
            uint32_t af[4];
            ldsm_x4_t(af, abase + (uint32_t)((16 * kk * LH + 16 * mt) * 2));
            mma_f16(sv[mt], af, {bq[2 * half], bq[2 * half + 1]});
          }
        }
      }
#pragma unroll
      for (int mt = 0; mt < MT2; ++mt)
#pragma unroll
        for (int hi = 0; hi < 2; ++hi) {
          const int r = m2 + 16 * mt + g + 8 * hi, j = n2 + 2 * t;
          const float e = eb[s * D + r];
          float2 sp = *reinterpret_cast<const float2*>(S + r * LS + j);
          const float a0 = sv[mt][2 * hi], a1 = sv[mt][2 * hi + 1];
          if (BWD) {
            const float2 y = __half22float2(*reinterpret_cast<const __half2*>(Yb + (s * D + r) * CW + j));
            sp = make_float2(e * sp.x - a0 + y.x, e * sp.y - a1 + y.y);
          } else {
            sp = make_float2(e * sp.x + a0, e * sp.y + a1);
          }
          *reinterpret_cast<float2*>(S + r * LS + j) = sp;
          ST[j * LT + r] = __float2half_rn(sp.x);
          ST[(j + 1) * LT + r] = __float2half_rn(sp.y);
        }
    }
  }
  if (BWD && a.dS0) {
    __syncthreads();
    for (int idx = tid; idx < D * CW; idx += NT) {
      const int r = idx / CW, j = idx % CW;
      a.dS0[(bh * D + r) * D + c0 + j] = S[r * LS + j];
    }
  }
}

template <int D>
__global__ void __launch_bounds__(NT, 2) cbwd_chain_h_kernel(CbwdArgs a) {
  extern __shared__ __align__(16) uint8_t smh[];
  if (blockIdx.z & 1) chain_h_pass<D, true>(a, (int)(blockIdx.z >> 1), smh);
  else chain_h_pass<D, false>(a, (int)(blockIdx.z >> 1), smh);
}

// ---- contractions with the chunk's entry state and exit gradient -------------------------
template <int D>
constexpr size_t state_grad_smem() { return sizeof(float) * (2 * D * LDJ + 4 * CH * LDJ); }

template <int D, bool SPLIT>
__global__ void __launch_bounds__(NT) cbwd_state_grad_kernel(CbwdArgs a) {
  constexpr int NTD = D / 32;
  extern __shared__ __align__(16) float sm[];
  float* S0b = sm;              // [D][LDJ]  S columns j0 .. j0 + JB
  float* dSb = S0b + D * LDJ;   // [D][LDJ]  dS columns
  float* dOb = dSb + D * LDJ;   // [CH][LDJ]
  float* dUb = dOb + CH * LDJ;
  float* Ub = dUb + CH * LDJ;
  float* Vb = Ub + CH * LDJ;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, g = lane >> 2, t = lane & 3;
  const ChunkPos p = chunk_pos(a);
  const float* S = a.w.S + p.ch * D * D;
  const float* dS = a.w.dS + p.ch * D * D;
  const float* dU = a.w.dU + p.ch * CH * D;
  const float* U = a.w.U + p.ch * CH * D;
  // stage columns [j0, j0 + JB) of the chunk's operands; which ones per pass
  auto stage = [&](int j0, bool pass2) {
    __syncthreads();
    for (int idx = tid; idx < D * JB / 4; idx += NT) {
      const int r = idx / (JB / 4), c4 = (idx % (JB / 4)) * 4;
      if (!pass2) *reinterpret_cast<float4*>(S0b + r * LDJ + c4) = *reinterpret_cast<const float4*>(S + r * D + j0 + c4);
      *reinterpret_cast<float4*>(dSb + r * LDJ + c4) = *reinterpret_cast<const float4*>(dS + r * D + j0 + c4);
    }
    for (int idx = tid; idx < CH * JB / 4; idx += NT) {
      const int r = idx / (JB / 4), c4 = (idx % (JB / 4)) * 4;
      const bool in = r < p.n;
      const int64_t tk = (p.tok0 + (int64_t)r * a.H) * D + j0 + c4;
      float4 o4 = make_float4(0.f, 0.f, 0.f, 0.f);
      if (in) o4 = make_float4(ld_act(a.d_o, tk, a.bf16), ld_act(a.d_o, tk + 1, a.bf16), ld_act(a.d_o, tk + 2, a.bf16),
                               ld_act(a.d_o, tk + 3, a.bf16));
      *reinterpret_cast<float4*>(dOb + r * LDJ + c4) = o4;
      *reinterpret_cast<float4*>(dUb + r * LDJ + c4) = *reinterpret_cast<const float4*>(dU + r * D + j0 + c4);
      if (pass2) {
        *reinterpret_cast<float4*>(Ub + r * LDJ + c4) = *reinterpret_cast<const float4*>(U + r * D + j0 + c4);
        *reinterpret_cast<float4*>(Vb + r * LDJ + c4) =
            in ? *reinterpret_cast<const float4*>(a.v + tk) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    __syncthreads();
  };
  const int m0 = 32 * (warp & 1), n0 = (D / 4) * (warp >> 1);        // CH x D blocks
  const int p0 = 16 * (warp & 3), q0 = 32 * (warp >> 2);             // CH x CH blocks
  {  // dQG = dO S^T, dW = -dU S^T, and rowsum(dS o S)
    float aq[2][NTD][4], aw[2][NTD][4];
    zero4(aq);
    zero4(aw);
    float lastp = 0.f;
    for (int j0 = 0; j0 < D; j0 += JB) {
      stage(j0, false);
      wmma3<2, NTD, false, SPLIT>(aq, dOb, LDJ, 1, S0b, 1, LDJ, JB, m0, n0, lane);
      wmma3<2, NTD, false, SPLIT>(aw, dUb, LDJ, 1, S0b, 1, LDJ, JB, m0, n0, lane);
      if (tid < D)
#pragma unroll 8
        for (int j = 0; j < JB; ++j) lastp = fmaf(dSb[tid * LDJ + j], S0b[tid * LDJ + j], lastp);
    }
    float* dQG = a.w.dQG + p.ch * CH * D;
    float* dW = a.w.dW + p.ch * CH * D;
    FRAG_LOOP(2, NTD) {
      const int r = FRAG_R(m0), c = FRAG_C(n0);
      dQG[r * D + c] = aq[mt][nt][i];
      dW[r * D + c] = -aw[mt][nt][i];
    }
    if (tid < D) a.w.last[p.ch * D + tid] = lastp * a.w.egl[p.ch * D + tid];
  }
  {  // dKt = U dS^T, dP = lower(dO U^T), dU V^T
    float ak[2][NTD][4], ap[1][4][4], auv[1][4][4];
    zero4(ak);
    zero4(ap);
    zero4(auv);
    for (int j0 = 0; j0 < D; j0 += JB) {
      stage(j0, true);
      wmma3<2, NTD, false, SPLIT>(ak, Ub, LDJ, 1, dSb, 1, LDJ, JB, m0, n0, lane);
      wmma3<1, 4, false, SPLIT>(ap, dOb, LDJ, 1, Ub, 1, LDJ, JB, p0, q0, lane);
      wmma3<1, 4, false, SPLIT>(auv, dUb, LDJ, 1, Vb, 1, LDJ, JB, p0, q0, lane);
    }
    float* dKt = a.w.dKt + p.ch * CH * D;
    float* dP = a.w.dP + p.ch * CH * CH;
    float* dUV = a.w.dUV + p.ch * CH * CH;
    FRAG_LOOP(2, NTD) dKt[FRAG_R(m0) * D + FRAG_C(n0)] = ak[mt][nt][i];
    FRAG_LOOP(1, 4) {
      const int r = FRAG_R(p0), c = FRAG_C(q0);
      dP[r * CH + c] = c <= r ? ap[mt][nt][i] : 0.f;
      dUV[r * CH + c] = auv[mt][nt][i];
    }
  }
}

// ---- the chunk-local part of the adjoint ---------------------------------------------
template <int D>
constexpr size_t local_grad_smem() { return sizeof(float) * (4 * CH * (D + 4) + 5 * CH * LDC + 5 * D + 2 * CH); }

template <int D, bool SPLIT>
__global__ void __launch_bounds__(NT, 1) cbwd_local_grad_kernel(CbwdArgs a) {
  constexpr int LDD = D + 4, NTD = D / 32;
  extern __shared__ __align__(16) float sm[];
  float* Gs = sm;                 // [CH][LDD] g, then E = e^{g - g_m}, at the end dg
  float* Kx = Gs + CH * LDD;      // k e^{g - g_m}
  float* Fs = Kx + CH * LDD;      // dW e^{g_m}, later q e^{g - g_m}
  float* Bs = Fs + CH * LDD;      // dU, later k e^{g_m - g}
  float* Xs = Bs + CH * LDD;      // [CH][LDC] X
  float* dTs = Xs + CH * LDC;     // dT
  float* Ms = dTs + CH * LDC;     // X^T dT Diag(beta)
  float* dPs = Ms + CH * LDC;     // dP
  float* Abs = dPs + CH * LDC;    // A / beta, later Diag(beta) dA
  float* gm = Abs + CH * LDC;     // [D]
  float* gl = gm + D;             // [D]
  float* egm = gl + D;            // [D] e^{g_m}
  float* eglm = egm + D;          // [D] e^{g_l - g_m}
  float* colk = eglm + D;         // [D] column sums of dKt o Kt
  float* bs = colk + D;           // [CH]
  float* db = bs + CH;            // [CH] dbeta
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, g = lane >> 2, t = lane & 3;
  const ChunkPos p = chunk_pos(a);
  const int64_t rs = (int64_t)a.H * D;
  const float* q = a.q + p.tok0 * D;
  const float* k = a.k + p.tok0 * D;
  const int64_t cd = p.ch * CH * D, cc = p.ch * CH * CH;
  const int m0 = 32 * (warp & 1), n0 = (D / 4) * (warp >> 1);        // CH x D blocks
  const int p0 = 16 * (warp & 3), q0 = 32 * (warp >> 2);             // CH x CH blocks

  // every input tile of the chunk in flight together (k lands raw in Kx, dW in Fs)
  stage_rows<D>(Gs, LDD, a.la + p.tok0 * D, rs, p.n, tid);
  stage_rows<D>(Kx, LDD, k, rs, p.n, tid);
  stage_rows<D>(Fs, LDD, a.w.dW + cd, D, CH, tid);
  stage_rows<D>(Bs, LDD, a.w.dU + cd, D, CH, tid);
  stage_rows<CH>(Xs, LDC, a.w.X + cc, CH, CH, tid);
  stage_rows<CH>(dTs, LDC, a.w.dUV + cc, CH, CH, tid);
  stage_rows<CH>(dPs, LDC, a.w.dP + cc, CH, CH, tid);
  stage_rows<CH>(Abs, LDC, a.w.Ab + cc, CH, CH, tid);
  cp_async_commit();
  if (tid < CH) bs[tid] = tid < p.n ? ld_act(a.beta, p.tok0 + (int64_t)tid * a.H, a.bf16) : 0.f;
  if (tid < D) colk[tid] = 0.f;
  cp_async_wait_all();
  __syncthreads();
  chunk_cumsum<D>(Gs, gm, gl, egm, eglm, tid);
  __syncthreads();
  // in place: E = e^{g - g_m} replaces g (every later use of g is through E and 1/E),
  // Kx = k E, Fs = dW e^{g_m}
  for (int idx = tid; idx < CH * D / 4; idx += NT) {
    const int r = idx / (D / 4), c4 = (idx % (D / 4)) * 4;
    float* ep = Gs + r * LDD + c4;
    float* kp = Kx + r * LDD + c4;
    float* fp = Fs + r * LDD + c4;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float e = expf(ep[j] - gm[c4 + j]);
      ep[j] = e;
      kp[j] *= e;
      fp[j] *= egm[c4 + j];
    }
  }
  __syncthreads();
  {  // dT = dW KG^T + dU V^T
    float tt[1][4][4];
    zero4(tt);
    wmma3<1, 4, false, SPLIT>(tt, Fs, LDD, 1, Kx, 1, LDD, D, p0, q0, lane);
    FRAG_LOOP(1, 4) dTs[FRAG_R(p0) * LDC + FRAG_C(q0)] += tt[mt][nt][i];
  }
  // this thread's elements of dq, dk and dg (the CH x D block tiling)
  float dq[2][NTD][4], dk[2][NTD][4], dg[2][NTD][4];
  {  // dv = Diag(beta) X^T dU
    float acc[2][NTD][4];
    zero4(acc);
    wmma3<2, NTD, false, SPLIT>(acc, Xs, 1, LDC, Bs, LDD, 1, CH, m0, n0, lane);
    FRAG_LOOP(2, NTD) {
      const int r = FRAG_R(m0);
      if (r < p.n) a.dv[(p.tok0 + (int64_t)r * a.H) * D + FRAG_C(n0)] = bs[r] * acc[mt][nt][i];
    }
  }
  {  // dKG = Diag(beta) X^T dW; the dq, dk, dg terms of KG, QG and Kt
    float acc[2][NTD][4];
    zero4(acc);
    wmma3<2, NTD, false, SPLIT>(acc, Xs, 1, LDC, Fs, LDD, 1, CH, m0, n0, lane);
    const float* dKt = a.w.dKt + cd;
    const float* dQG = a.w.dQG + cd;
#pragma unroll
    for (int nt = 0; nt < NTD; ++nt)
#pragma unroll
      for (int par = 0; par < 2; ++par) {
        float ck = 0.f;
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
          for (int hi = 0; hi < 2; ++hi) {
            const int i = 2 * hi + par;
            const int r = FRAG_R(m0), c = FRAG_C(n0);
            const bool in = r < p.n;
            const float e1 = Gs[r * LDD + c];
            const float e2 = eglm[c] * __fdividef(1.f, e1), eg = egm[c] * e1;   // e^{g_l - g}, e^{g}
            const float kv = in ? k[r * rs + c] : 0.f, qv = in ? q[r * rs + c] : 0.f;
            const float dkt = dKt[r * D + c], dqg = dQG[r * D + c];
            const float av = bs[r] * acc[mt][nt][i] * e1;   // dKG o e^g
            dk[mt][nt][i] = av + dkt * e2;
            dq[mt][nt][i] = dqg * eg;
            dg[mt][nt][i] = kv * av - kv * e2 * dkt + qv * eg * dqg;
            ck = fmaf(kv * e2, dkt, ck);
          }
        atomicAdd(&colk[n0 + 8 * nt + 2 * t + par], ck);
      }
  }
  __syncthreads();   // dT complete; the products reading Fs and Bs are done
  stage_rows<D>(Fs, LDD, q, rs, p.n, tid);   // raw q and k, scaled below
  stage_rows<D>(Bs, LDD, k, rs, p.n, tid);
  cp_async_commit();
  {  // M = X^T dT Diag(beta); the first dbeta term, colsum(X o dT)
    float m[1][4][4];
    zero4(m);
    wmma3<1, 4, false, SPLIT>(m, Xs, 1, LDC, dTs, LDC, 1, CH, p0, q0, lane);
    FRAG_LOOP(1, 4) {
      const int c = FRAG_C(q0);
      Ms[FRAG_R(p0) * LDC + c] = m[mt][nt][i] * bs[c];
    }
    if (tid < CH) {
      float s = 0.f;
      for (int r = 0; r < CH; ++r) s = fmaf(Xs[r * LDC + tid], dTs[r * LDC + tid], s);
      db[tid] = s;
    }
  }
  // q e^{g - g_m} and k e^{g_m - g} replace dW e^{g_m} and dU, whose products are done
  cp_async_wait_all();
  __syncthreads();
  for (int idx = tid; idx < CH * D / 4; idx += NT) {
    const int r = idx / (D / 4), c4 = (idx % (D / 4)) * 4;
    float* fp = Fs + r * LDD + c4;
    float* bp = Bs + r * LDD + c4;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float e = Gs[r * LDD + c4 + j];
      fp[j] *= e;
      bp[j] *= __fdividef(1.f, e);
    }
  }
  __syncthreads();
  {  // dA = -strict(M X^T); the second dbeta term, rowsum(dA o A/beta); dAb = Diag(beta) dA
    float m[1][4][4];
    zero4(m);
    wmma3<1, 4, false, SPLIT>(m, Ms, LDC, 1, Xs, 1, LDC, CH, p0, q0, lane);
#pragma unroll
    for (int hi = 0; hi < 2; ++hi) {
      const int r = p0 + g + 8 * hi;
      float part = 0.f;
#pragma unroll
      for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int par = 0; par < 2; ++par) {
          const int c = q0 + 8 * nt + 2 * t + par;
          const float dA = c < r ? -m[0][nt][2 * hi + par] : 0.f;
          part = fmaf(dA, Abs[r * LDC + c], part);
          Abs[r * LDC + c] = dA * bs[r];
        }
      atomicAdd(&db[r], part);
    }
  }
  __syncthreads();
  if (tid < p.n) a.dbeta[p.tok0 + (int64_t)tid * a.H] = db[tid];
  {  // R2 = e^{g - g_m} o (dP KN): dq, and R1 = e^{g - g_m} o (dAb KN): dk
    float acc[2][NTD][4];
    zero4(acc);
    wmma3<2, NTD, false, SPLIT>(acc, dPs, LDC, 1, Bs, LDD, 1, CH, m0, n0, lane);
    FRAG_LOOP(2, NTD) {
      const int r = FRAG_R(m0), c = FRAG_C(n0);
      const float r2 = acc[mt][nt][i] * Gs[r * LDD + c];
      const float qv = r < p.n ? q[r * rs + c] : 0.f;
      dq[mt][nt][i] += r2;
      dg[mt][nt][i] = fmaf(qv, r2, dg[mt][nt][i]);
    }
    zero4(acc);
    wmma3<2, NTD, false, SPLIT>(acc, Abs, LDC, 1, Bs, LDD, 1, CH, m0, n0, lane);
    FRAG_LOOP(2, NTD) {
      const int r = FRAG_R(m0), c = FRAG_C(n0);
      const float r1 = acc[mt][nt][i] * Gs[r * LDD + c];
      const float kv = r < p.n ? k[r * rs + c] : 0.f;
      dk[mt][nt][i] += r1;
      dg[mt][nt][i] = fmaf(kv, r1, dg[mt][nt][i]);
    }
  }
  {  // R3 = e^{g_m - g} o (dAb^T Kx + dP^T Qx): dk
    float acc[2][NTD][4];
    zero4(acc);
    wmma3<2, NTD, false, SPLIT>(acc, Abs, 1, LDC, Kx, LDD, 1, CH, m0, n0, lane);
    wmma3<2, NTD, false, SPLIT>(acc, dPs, 1, LDC, Fs, LDD, 1, CH, m0, n0, lane);
    FRAG_LOOP(2, NTD) {
      const int r = FRAG_R(m0), c = FRAG_C(n0);
      const bool in = r < p.n;
      const float r3 = acc[mt][nt][i] * __fdividef(1.f, Gs[r * LDD + c]);
      const float kv = in ? k[r * rs + c] : 0.f;
      dk[mt][nt][i] += r3;
      dg[mt][nt][i] = fmaf(-kv, r3, dg[mt][nt][i]);
      if (in) {
        const int64_t tk = (p.tok0 + (int64_t)r * a.H) * D + c;
        a.dq[tk] = dq[mt][nt][i];
        a.dk[tk] = dk[mt][nt][i];
      }
    }
  }
  __syncthreads();   // every read of g is done: Gs takes dg
  FRAG_LOOP(2, NTD) Gs[FRAG_R(m0) * LDD + FRAG_C(n0)] = dg[mt][nt][i];
  __syncthreads();
  if (tid < D) {   // dlog alpha = reverse running sum of dg; the exit terms enter at the last row
    float s = colk[tid] + a.w.last[p.ch * D + tid];
    for (int r = CH - 1; r >= 0; --r) {
      s += Gs[r * LDD + tid];
      if (r < p.n) a.dla[(p.tok0 + (int64_t)r * a.H) * D + tid] = s;
    }
  }
}

template <typename T>
__global__ void bwd_beta_kernel(const float* src, T* dst, int64_t n) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) dst[i] = from_f32<T>(src[i]);
}

// ---- conv backward, text tokens --------------------------------------------------
// (the visual tokens' dx and dw run on the forward conv's tiles: launch_shortconv_bwd_vis)
struct ConvBwdArgs {
  const void* x[3];          // raw inputs, dtype [B][N][C]
  const float* dy[3];        // gradients of the conv outputs, fp32 [B][N][C]
  void* dx[3];               // dtype [B][N][C]
  const float* w_text;       // [3][C][text_k]
  float* dw_text;            // [3][C][text_k], accumulated
  int64_t N, L;
  int B, C, text_k;
};

// A CTA covers CB_TOK text tokens of one batch item and 32 channels of one tensor (one per
// lane; 8 warps split the tokens), the channel's taps in registers.
constexpr int CB_TOK = 256;

// dx = every text output that read x, times its tap weight (the transpose of the causal conv)
template <typename T>
__global__ void __launch_bounds__(256) conv_bwd_dx_kernel(ConvBwdArgs a) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, tensor = blockIdx.z;
  const int c = blockIdx.y * 32 + lane;
  const int64_t bpi = (a.L + CB_TOK - 1) / CB_TOK;
  const int64_t b = blockIdx.x / bpi, n0 = (blockIdx.x % bpi) * CB_TOK;
  float wt[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) wt[i] = i < a.text_k ? a.w_text[((int64_t)tensor * a.C + c) * a.text_k + i] : 0.f;
  const float* dy = (tensor == 0 ? a.dy[0] : tensor == 1 ? a.dy[1] : a.dy[2]) + b * a.N * a.C + c;
  T* dx = static_cast<T*>(tensor == 0 ? a.dx[0] : tensor == 1 ? a.dx[1] : a.dx[2]) + b * a.N * a.C + c;
  const int64_t n1 = min(n0 + CB_TOK, a.L);
  for (int64_t n = n0 + warp; n < n1; n += 8) {
    // y[m] reads x[m - (K-1) + j]: x[n] feeds the text outputs m = n + K-1-j < L
    float acc = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int64_t m = n + (a.text_k - 1) - j;
      if (j < a.text_k && m < a.L) acc += wt[j] * dy[m * a.C];
    }
    dx[n * a.C] = from_f32<T>(acc);
  }
}

// dw_text = sum over text tokens of x * dy per channel and tap: per-warp sums meet in shared
// memory, then one atomic add per (channel, tap) and CTA
template <typename TIn>
__global__ void __launch_bounds__(256) conv_bwd_dw_kernel(ConvBwdArgs a) {
  __shared__ float part[8][8][32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, tensor = blockIdx.z;
  const int c = blockIdx.y * 32 + lane;
  const int64_t bpi = (a.L + CB_TOK - 1) / CB_TOK;
  const int64_t b = blockIdx.x / bpi, n0 = (blockIdx.x % bpi) * CB_TOK;
  const TIn* x = static_cast<const TIn*>(tensor == 0 ? a.x[0] : tensor == 1 ? a.x[1] : a.x[2]) + b * a.N * a.C + c;
  const float* dy = (tensor == 0 ? a.dy[0] : tensor == 1 ? a.dy[1] : a.dy[2]) + b * a.N * a.C + c;
  float at[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) at[i] = 0.f;
  const int64_t n1 = min(n0 + CB_TOK, a.L);
  for (int64_t n = n0 + warp; n < n1; n += 8) {
    const float gv = dy[n * a.C];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int64_t s = n - (a.text_k - 1) + j;
      if (j < a.text_k && s >= 0) at[j] += to_f32(x[s * a.C]) * gv;
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) part[warp][i][lane] = at[i];
  __syncthreads();
  if (warp < a.text_k) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) s += part[w][warp][lane];
    atomicAdd(a.dw_text + ((int64_t)tensor * a.C + c) * a.text_k + warp, s);
  }
}

struct BwdLayout {
  size_t act32, dbeta, cd, cc, dd, d1, total;
  int nc;
};

// workspace: status word, q', k', v', dq', dk', dv' (fp32), dbeta (fp32), then the per
// chunk-head arrays of CbwdBufs
BwdLayout bwd_layout(const Dims& d) {
  BwdLayout l;
  const size_t elems = (size_t)d.B * d.N * d.H * d.dk;
  l.act32 = align256(elems * sizeof(float));
  l.dbeta = align256((size_t)d.B * d.N * d.H * sizeof(float));
  l.nc = (int)((d.N + CH - 1) / CH);
  const size_t nch = (size_t)d.B * d.H * l.nc;
  l.cd = align256(nch * CH * d.dk * sizeof(float));
  l.cc = align256(nch * CH * CH * sizeof(float));
  l.dd = align256(nch * d.dk * d.dk * sizeof(float));
  l.d1 = align256(nch * d.dk * sizeof(float));
  l.total = 256 + 6 * l.act32 + l.dbeta + 9 * l.cd + 4 * l.cc + 3 * l.dd + 2 * l.d1;
  return l;
}

CbwdBufs carve(const BwdLayout& l, char* p) {
  CbwdBufs w;
  float** cd[] = {&w.W, &w.Ut, &w.Kt, &w.Z, &w.U, &w.dU, &w.dQG, &w.dW, &w.dKt};
  for (float** x : cd) { *x = reinterpret_cast<float*>(p); p += l.cd; }
  float** cc[] = {&w.X, &w.Ab, &w.dP, &w.dUV};
  for (float** x : cc) { *x = reinterpret_cast<float*>(p); p += l.cc; }
  float** dd[] = {&w.Y, &w.S, &w.dS};
  for (float** x : dd) { *x = reinterpret_cast<float*>(p); p += l.dd; }
  w.egl = reinterpret_cast<float*>(p); p += l.d1;
  w.last = reinterpret_cast<float*>(p);
  return w;
}

template <typename K>
cudaError_t set_smem(K kernel, size_t bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

// SPLIT: every product at fp32 accuracy (fp32 problems: split tf32 products, fp32 chain
// operands).  bf16 problems take one tf32 product of rounded operands in the per-chunk kernels and
// fp16 operands in the chains, which run together in one launch.
template <int D, bool SPLIT>
cudaError_t launch_scan_bwd(const CbwdArgs& a, const Dims& d, cudaStream_t s) {
  cudaError_t e;
  const dim3 chunks((unsigned)a.nc, (unsigned)d.H, (unsigned)d.B);
  const dim3 cols((unsigned)(D / CW), (unsigned)d.H, (unsigned)d.B);
  if ((e = set_smem(cbwd_prep_kernel<D, SPLIT>, prep_smem<D>())) != cudaSuccess) return e;
  cbwd_prep_kernel<D, SPLIT><<<chunks, NT, prep_smem<D>(), s>>>(a);
  if (SPLIT) {
    if ((e = set_smem(cbwd_chain_kernel<D, false>, chain_smem<D, false>())) != cudaSuccess) return e;
    cbwd_chain_kernel<D, false><<<cols, NT, chain_smem<D, false>(), s>>>(a);
    if ((e = set_smem(cbwd_chain_kernel<D, true>, chain_smem<D, true>())) != cudaSuccess) return e;
    cbwd_chain_kernel<D, true><<<cols, NT, chain_smem<D, true>(), s>>>(a);
  } else {
    const dim3 both((unsigned)(D / CW), (unsigned)d.H, (unsigned)(2 * d.B));
    if ((e = set_smem(cbwd_chain_h_kernel<D>, chain_h_smem<D>())) != cudaSuccess) return e;
    cbwd_chain_h_kernel<D><<<both, NT, chain_h_smem<D>(), s>>>(a);
  }
  if ((e = set_smem(cbwd_state_grad_kernel<D, SPLIT>, state_grad_smem<D>())) != cudaSuccess) return e;
  cbwd_state_grad_kernel<D, SPLIT><<<chunks, NT, state_grad_smem<D>(), s>>>(a);
  if ((e = set_smem(cbwd_local_grad_kernel<D, SPLIT>, local_grad_smem<D>())) != cudaSuccess) return e;
  cbwd_local_grad_kernel<D, SPLIT><<<chunks, NT, local_grad_smem<D>(), s>>>(a);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_conv_bwd(const ConvBwdArgs& c, const Dims& d, cudaStream_t s) {
  if (d.L <= 0) return cudaSuccess;
  const dim3 grid((unsigned)(d.B * ((d.L + CB_TOK - 1) / CB_TOK)), (unsigned)(c.C / 32), 3);
  conv_bwd_dx_kernel<T><<<grid, 256, 0, s>>>(c);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  conv_bwd_dw_kernel<T><<<grid, 256, 0, s>>>(c);
  return cudaGetLastError();
}

}  // namespace

size_t bwd_workspace_bytes(const Dims& d, kda_dtype) { return bwd_layout(d).total; }

cudaError_t launch_bwd(const Dims& d, kda_dtype dt, const void* q, const void* k, const void* v,
                       const float* log_alpha, const void* beta, const float* w_text, const float* w_vis,
                       const float* S0, const void* d_o, const float* dSN, void* dq, void* dk, void* dv,
                       float* dla, void* dbeta, float* dw_text, float* dw_vis, float* dS0, void* ws,
                       cudaStream_t s, int* launches) {
  const BwdLayout l = bwd_layout(d);
  char* base = static_cast<char*>(ws) + 256;
  float* act[6];
  for (int i = 0; i < 6; ++i) act[i] = reinterpret_cast<float*>(base + i * l.act32);   // q', k', v', dq', dk', dv'
  float* dbeta32 = reinterpret_cast<float*>(base + 6 * l.act32);
  const int C = d.H * d.dk;
  cudaError_t e;
  if ((e = cudaMemsetAsync(dw_text, 0, sizeof(float) * 3 * C * d.text_k, s)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(dw_vis, 0, sizeof(float) * 3 * C * 27, s)) != cudaSuccess) return e;
  if (d.N == 0) {
    if (!dS0) return cudaSuccess;
    const size_t bytes = (size_t)d.B * d.H * d.dk * d.dv * sizeof(float);
    return dSN ? cudaMemcpyAsync(dS0, dSN, bytes, cudaMemcpyDeviceToDevice, s) : cudaMemsetAsync(dS0, 0, bytes, s);
  }
  // 1. the convolved activations, fp32
  if ((e = launch_shortconv(d, dt, q, k, v, w_text, w_vis, act[0], act[1], act[2], s, launches, false, true)) !=
      cudaSuccess)
    return e;
  // 2. scan backward, chunked
  CbwdArgs a;
  a.q = act[0]; a.k = act[1]; a.v = act[2]; a.la = log_alpha; a.beta = beta; a.d_o = d_o; a.S0 = S0; a.dSN = dSN;
  a.dq = act[3]; a.dk = act[4]; a.dv = act[5]; a.dla = dla; a.dbeta = dbeta32; a.dS0 = dS0;
  a.w = carve(l, base + 6 * l.act32 + l.dbeta);
  a.N = d.N; a.H = d.H; a.nc = l.nc; a.bf16 = dt == KDA_DT_BF16;
  a.status = static_cast<uint32_t*>(ws);
  if (a.bf16) e = d.dk == 128 ? launch_scan_bwd<128, false>(a, d, s) : launch_scan_bwd<64, false>(a, d, s);
  else e = d.dk == 128 ? launch_scan_bwd<128, true>(a, d, s) : launch_scan_bwd<64, true>(a, d, s);
  if (e != cudaSuccess) return e;
  const int64_t nb = (int64_t)d.B * d.N * d.H;
  if (dt == KDA_DT_BF16)
    bwd_beta_kernel<__nv_bfloat16><<<(unsigned)((nb + 255) / 256), 256, 0, s>>>(dbeta32, static_cast<__nv_bfloat16*>(dbeta), nb);
  else
    bwd_beta_kernel<float><<<(unsigned)((nb + 255) / 256), 256, 0, s>>>(dbeta32, static_cast<float*>(dbeta), nb);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // 3. conv backward: text tokens here, visual tokens on the forward conv's tiles
  ConvBwdArgs c;
  c.x[0] = q; c.x[1] = k; c.x[2] = v;
  c.dy[0] = act[3]; c.dy[1] = act[4]; c.dy[2] = act[5];
  c.dx[0] = dq; c.dx[1] = dk; c.dx[2] = dv;
  c.w_text = w_text; c.dw_text = dw_text;
  c.N = d.N; c.L = d.L; c.B = d.B; c.C = C; c.text_k = d.text_k;
  e = dt == KDA_DT_BF16 ? launch_conv_bwd<__nv_bfloat16>(c, d, s) : launch_conv_bwd<float>(c, d, s);
  if (e != cudaSuccess) return e;
  if ((e = launch_shortconv_bwd_vis(d, dt, c.x, c.dy, c.dx, w_vis, dw_vis, s, launches)) != cudaSuccess) return e;
  if (launches) *launches += 5 + 1 + (d.L > 0 ? 2 : 0);
  return cudaSuccess;
}

}  // namespace kda
