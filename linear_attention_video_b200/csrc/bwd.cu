// Backward pass of the modality-aware short convolution + KDA scan: the
// gradients of kda_fwd's outputs (o and the final state) with respect to q, k,
// v, log alpha, beta, the conv weights and the initial state.  fp32 on the CUDA
// cores.
//
// Forward step per head (paper.rainbus.top, section 方法步骤详情, step (5)),
// with S~ = Diag(alpha_t) S_{t-1}:
//     u = beta_t (v_t - S~^T k_t),   S_t = S~ + k_t u^T,   o_t = S_t^T q_t.
// Its adjoint, with dS the gradient reaching S_t from later tokens and
// G = dS + q_t do_t^T:
//     dq_t = S_t do_t,  du = G^T k_t,  dv_t = beta_t du,  dbeta_t = du . (v_t - S~^T k_t),
//     dk_t = G u - beta_t S~ du,  dS~ = G - beta_t k_t du^T,
//     dlog_alpha_t = rowsum(dS~ o S~),  dS_{t-1} = Diag(alpha_t) dS~.
// Column j of S only sees column j of v, so a CTA owns CWB value columns of
// one (batch item, head); the column sums of dq, dk, dlog alpha and dbeta are
// accumulated across CTAs with fp32 reductions in global memory.
//
// Kernels, in launch order:
//   conv (forward, fp32 out)  q', k', v' recomputed from the raw inputs
//   bwd_states_kernel         forward recurrence, the state stored every KC tokens
//   bwd_scan_kernel           per KC-token chunk in reverse: its states recomputed
//                             from the stored one into shared memory, then the
//                             adjoint token by token
//   bwd_beta_kernel           dbeta fp32 -> dtype
//   conv_bwd_dx_kernel        dx = transpose of the conv applied to dq', dk', dv'
//   conv_bwd_dw_kernel        dw = sum over tokens of x * dy, per channel and tap
#include "common.cuh"

#include <cuda_fp16.h>

namespace kda {
namespace {

constexpr int CWB = 8;    // value columns per CTA of the scan kernels (two CTAs share an SM)
constexpr int KC = 8;     // tokens between stored states (and per pipelined chunk of the adjoint kernel)

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

__device__ __forceinline__ float ld_act(const void* p, int64_t i, bool bf16) {
  return bf16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(p)[i]) : static_cast<const float*>(p)[i];
}

struct ScanBwdArgs {
  const float* q; const float* k; const float* v;   // convolved activations, fp32 [B][N][H][D]
  const float* la;                                   // [B][N][H][D]
  const void* beta;                                  // [B][N][H], dtype
  const float* S0;                                   // [B][H][D][D] or null
  const void* d_o;                                   // [B][N][H][D], dtype
  const float* dSN;                                  // [B][H][D][D] or null
  float* ckpt;                                       // [B][H][n_ck][D][D]: state before token KC c
  float* dq; float* dk; float* dv;                   // fp32 [B][N][H][D]; dq, dk accumulated
  float* dla;                                        // fp32 [B][N][H][D], accumulated
  float* dbeta;                                      // fp32 [B][N][H], accumulated
  float* dS0;                                        // [B][H][D][D] or null
  int64_t N; int H; int n_ck; bool bf16;
};

// Barrier over the DK threads of one row group: the whole CTA (id 0) or a named barrier.
template <int DK>
__device__ __forceinline__ void group_sync(int id) {
  if (id == 0) __syncthreads();
  else asm volatile("bar.sync %0, %1;" :: "r"(id), "r"(DK) : "memory");
}

// out[j] = sum over a row group's DK threads (row i) of x[j], for the CWB columns; every thread gets all
template <int DK>
__device__ __forceinline__ void colsum(const float (&x)[CWB], float* red, float* red2, float (&out)[CWB], int i,
                                       int bar) {
#pragma unroll
  for (int j = 0; j < CWB; ++j) red[i * (CWB + 1) + j] = x[j];
  group_sync<DK>(bar);
  const int j = i % CWB, part = i / CWB;   // DK / CWB parts of CWB rows
  float s = 0.f;
#pragma unroll
  for (int r = 0; r < CWB; ++r) s += red[(part * CWB + r) * (CWB + 1) + j];
#pragma unroll
  for (int off = CWB; off < 32; off <<= 1) s += __shfl_xor_sync(0xffffffffu, s, off);   // parts of one warp
  if ((i & 31) < CWB) red2[(i >> 5) * CWB + j] = s;
  group_sync<DK>(bar);
#pragma unroll
  for (int jj = 0; jj < CWB; ++jj) {
    float acc = 0.f;
#pragma unroll
    for (int w = 0; w < DK / 32; ++w) acc += red2[w * CWB + jj];
    out[jj] = acc;
  }
}

// Per-token inputs of one KC-token chunk, staged in shared memory: the row of
// each key channel (thread i loads element i of every token) and the CTA's
// value columns.  Loads for the next chunk are issued into registers before
// the current chunk is processed, so their latency overlaps its work.
template <int DK, int L = KC>
struct ChunkIn {
  float la[L][DK], k[L][DK], q[L][DK];
  float v[L][CWB], dout[L][CWB], beta[L];
};

template <int DK, int L = KC>
struct ChunkRegs {
  float la[L], k[L], q[L], v[L], dout[L], beta;
};

// thread i: element i of the chunk's rows (zero past the sequence end); threads < CWB also
// the CTA's value columns, threads < KC the gates
template <int DK, bool BWD, int L = KC>
__device__ __forceinline__ void load_chunk(const ScanBwdArgs& a, int b, int h, int c0, int64_t t0,
                                           ChunkRegs<DK, L>& r, int i) {
#pragma unroll
  for (int tau = 0; tau < L; ++tau) {
    const bool in = t0 + tau < a.N;
    const int64_t tok = ((int64_t)b * a.N + (in ? t0 + tau : 0)) * a.H + h;
    r.la[tau] = in ? a.la[tok * DK + i] : 0.f;
    r.k[tau] = in ? a.k[tok * DK + i] : 0.f;
    if (BWD) r.q[tau] = in ? a.q[tok * DK + i] : 0.f;
    if (i < CWB) {
      r.v[tau] = in ? a.v[tok * DK + c0 + i] : 0.f;
      if (BWD) r.dout[tau] = in ? ld_act(a.d_o, tok * DK + c0 + i, a.bf16) : 0.f;
    }
  }
  if (i < L) {
    const bool in = t0 + i < a.N;
    r.beta = in ? ld_act(a.beta, ((int64_t)b * a.N + t0 + i) * a.H + h, a.bf16) : 0.f;
  }
}

template <int DK, bool BWD, int L = KC>
__device__ __forceinline__ void store_chunk(const ChunkRegs<DK, L>& r, ChunkIn<DK, L>& c, int i) {
#pragma unroll
  for (int tau = 0; tau < L; ++tau) {
    c.la[tau][i] = r.la[tau];
    c.k[tau][i] = r.k[tau];
    if (BWD) c.q[tau][i] = r.q[tau];
    if (i < CWB) {
      c.v[tau][i] = r.v[tau];
      if (BWD) c.dout[tau][i] = r.dout[tau];
    }
  }
  if (i < L) c.beta[i] = r.beta;
}

template <int DK>
__global__ void __launch_bounds__(DK) bwd_states_kernel(ScanBwdArgs a) {
  constexpr int SL = 2 * KC;   // tokens staged per step (two stored states per step)
  __shared__ ChunkIn<DK, SL> cin;
  __shared__ float red[DK * (CWB + 1)];
  __shared__ float red2[(DK / 32) * CWB];
  const int g = blockIdx.x, h = blockIdx.y, b = blockIdx.z, i = threadIdx.x;
  const int c0 = g * CWB;
  const int64_t srow = (((int64_t)b * a.H + h) * DK + i) * DK + c0;
  float S[CWB];
#pragma unroll
  for (int j = 0; j < CWB; ++j) S[j] = a.S0 ? a.S0[srow + j] : 0.f;
  float* ck = a.ckpt + ((int64_t)b * a.H + h) * a.n_ck * DK * DK;
  const int n_steps = (int)((a.N + SL - 1) / SL);
  ChunkRegs<DK, SL> nxt;
  load_chunk<DK, false, SL>(a, b, h, c0, 0, nxt, i);
  for (int c = 0; c < n_steps; ++c) {
    const int64_t t0 = (int64_t)c * SL;
    const int nt = (int)min((int64_t)SL, a.N - t0);
    __syncthreads();   // the previous step's inputs are no longer read
    store_chunk<DK, false, SL>(nxt, cin, i);
    __syncthreads();
    if (c + 1 < n_steps) load_chunk<DK, false, SL>(a, b, h, c0, t0 + SL, nxt, i);
    for (int tau = 0; tau < nt; ++tau) {
      if (tau % KC == 0) {   // the state entering tokens t0 + tau ..
        float4* dst = reinterpret_cast<float4*>(ck + (((t0 + tau) / KC) * DK + i) * DK + c0);
#pragma unroll
        for (int q4 = 0; q4 < CWB / 4; ++q4) dst[q4] = make_float4(S[4 * q4], S[4 * q4 + 1], S[4 * q4 + 2], S[4 * q4 + 3]);
      }
      const float al = expf(cin.la[tau][i]);
      const float ki = cin.k[tau][i];
      const float bt = cin.beta[tau];
      float x[CWB], sk[CWB];
#pragma unroll
      for (int j = 0; j < CWB; ++j) {
        S[j] *= al;
        x[j] = S[j] * ki;
      }
      colsum<DK>(x, red, red2, sk, i, 0);
#pragma unroll
      for (int j = 0; j < CWB; ++j) S[j] += ki * (bt * (cin.v[tau][j] - sk[j]));
    }
  }
}

// The adjoint kernel runs two row groups of DK threads: group 0 recomputes the states (and u, r)
// of chunk c - 1 from its stored entry state while group 1 applies the adjoint to chunk c, whose
// states group 0 recomputed in the previous step; the groups meet at one CTA barrier per chunk.
template <int DK>
struct ScanBwdSmem {
  float st[2][KC + 1][DK][CWB];   // per buffer: entry state, then the state after each token
  float ub[2][KC][CWB];           // u = beta (v - S~^T k)
  float rb[2][KC][CWB];           // v - S~^T k
  ChunkIn<DK> in[2];              // inputs of each group's current chunk
  float red[2][DK * (CWB + 1)];
  float red2[2][(DK / 32) * CWB];
};

template <int DK>
constexpr size_t scan_bwd_smem() { return sizeof(ScanBwdSmem<DK>); }

template <int DK>
__global__ void __launch_bounds__(2 * DK, 2) bwd_scan_kernel(ScanBwdArgs a) {
  extern __shared__ __align__(16) unsigned char smraw[];
  ScanBwdSmem<DK>& sm = *reinterpret_cast<ScanBwdSmem<DK>*>(smraw);
  const int grp = threadIdx.x / DK, i = threadIdx.x % DK;
  const int bar = 1 + grp;   // named barrier of the row group
  const int g = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int c0 = g * CWB;
  const int64_t srow = (((int64_t)b * a.H + h) * DK + i) * DK + c0;
  const float* ck = a.ckpt + ((int64_t)b * a.H + h) * a.n_ck * DK * DK;
  ChunkIn<DK>& cin = sm.in[grp];
  float* red = sm.red[grp];
  float* red2 = sm.red2[grp];
  float dS[CWB];   // group 1: gradient reaching the current chunk's exit state
#pragma unroll
  for (int j = 0; j < CWB; ++j) dS[j] = (grp == 1 && a.dSN) ? a.dSN[srow + j] : 0.f;
  // step it: group 0 recomputes chunk n_ck - 1 - it, group 1 differentiates chunk n_ck - it
  ChunkRegs<DK> nxt;   // both groups start with chunk n_ck - 1 (group 1 one step later)
  if (grp == 0) load_chunk<DK, false>(a, b, h, c0, (int64_t)(a.n_ck - 1) * KC, nxt, i);
  else load_chunk<DK, true>(a, b, h, c0, (int64_t)(a.n_ck - 1) * KC, nxt, i);
  for (int it = 0; it <= a.n_ck; ++it) {
    const int c = grp == 0 ? a.n_ck - 1 - it : a.n_ck - it;
    const bool active = grp == 0 ? it < a.n_ck : it >= 1;
    const int buf = grp == 0 ? (it & 1) : ((it - 1) & 1);
    if (active) {
      const int64_t t0 = (int64_t)c * KC;
      const int nt = (int)min((int64_t)KC, a.N - t0);
      group_sync<DK>(bar);   // the group's previous inputs are no longer read
      if (grp == 0) store_chunk<DK, false>(nxt, cin, i);
      else store_chunk<DK, true>(nxt, cin, i);
      group_sync<DK>(bar);
      if (c > 0) {
        if (grp == 0) load_chunk<DK, false>(a, b, h, c0, t0 - KC, nxt, i);
        else load_chunk<DK, true>(a, b, h, c0, t0 - KC, nxt, i);
      }
      float* st = &sm.st[buf][0][0][0];
      float* ub = &sm.ub[buf][0][0];
      float* rb = &sm.rb[buf][0][0];
      if (grp == 0) {
        // states of chunk c, recomputed from the stored entry state
        float S[CWB];
        const float* src = ck + ((int64_t)c * DK + i) * DK + c0;
#pragma unroll
        for (int j = 0; j < CWB; ++j) {
          S[j] = src[j];
          st[i * CWB + j] = S[j];
        }
        for (int tau = 0; tau < nt; ++tau) {
          const float al = expf(cin.la[tau][i]);
          const float ki = cin.k[tau][i];
          const float bt = cin.beta[tau];
          float x[CWB], sk[CWB];
#pragma unroll
          for (int j = 0; j < CWB; ++j) {
            S[j] *= al;
            x[j] = S[j] * ki;
          }
          colsum<DK>(x, red, red2, sk, i, bar);
          float* dst = st + ((size_t)(1 + tau) * DK + i) * CWB;
#pragma unroll
          for (int j = 0; j < CWB; ++j) {
            const float r = cin.v[tau][j] - sk[j];
            S[j] += ki * (bt * r);
            dst[j] = S[j];
            if (i == 0) {
              ub[tau * CWB + j] = bt * r;
              rb[tau * CWB + j] = r;
            }
          }
        }
      } else {
        // the adjoint over chunk c, token by token in reverse
        for (int tau = nt - 1; tau >= 0; --tau) {
          const int64_t tok = ((int64_t)b * a.N + t0 + tau) * a.H + h;
          const float al = expf(cin.la[tau][i]);
          const float ki = cin.k[tau][i];
          const float qi = cin.q[tau][i];
          const float bt = cin.beta[tau];
          const float* sp = st + ((size_t)tau * DK + i) * CWB;         // S_{t-1}
          const float* sc = st + ((size_t)(tau + 1) * DK + i) * CWB;   // S_t
          float sv[CWB], G[CWB], x[CWB], du[CWB];
          float dqi = 0.f;
#pragma unroll
          for (int j = 0; j < CWB; ++j) {
            const float doj = cin.dout[tau][j];
            sv[j] = al * sp[j];                 // S~
            G[j] = dS[j] + qi * doj;
            dqi += sc[j] * doj;
            x[j] = G[j] * ki;
          }
          atomicAdd(a.dq + tok * DK + i, dqi);
          colsum<DK>(x, red, red2, du, i, bar);
          if (i == 0) {
            float db = 0.f;
#pragma unroll
            for (int j = 0; j < CWB; ++j) db += du[j] * rb[tau * CWB + j];
            atomicAdd(a.dbeta + tok, db);
            float4* dvp = reinterpret_cast<float4*>(a.dv + tok * DK + c0);   // 32-byte aligned: c0 = 8 g
#pragma unroll
            for (int q4 = 0; q4 < CWB / 4; ++q4)
              dvp[q4] = make_float4(bt * du[4 * q4], bt * du[4 * q4 + 1], bt * du[4 * q4 + 2], bt * du[4 * q4 + 3]);
          }
          float dki = 0.f, dlai = 0.f;
#pragma unroll
          for (int j = 0; j < CWB; ++j) {
            const float dst = G[j] - bt * ki * du[j];   // dS~
            dki += G[j] * ub[tau * CWB + j] - bt * sv[j] * du[j];
            dlai += dst * sv[j];
            dS[j] = al * dst;
          }
          atomicAdd(a.dk + tok * DK + i, dki);
          atomicAdd(a.dla + tok * DK + i, dlai);
        }
      }
    }
    __syncthreads();   // group 0's states of this step are complete; group 1 is done with the other buffer
  }
  if (grp == 1 && a.dS0)
#pragma unroll
    for (int j = 0; j < CWB; ++j) a.dS0[srow + j] = dS[j];
}

template <typename T>
__global__ void bwd_beta_kernel(const float* src, T* dst, int64_t n) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) dst[i] = from_f32<T>(src[i]);
}

// ---- conv backward ------------------------------------------------------------
struct ConvBwdArgs {
  const void* x[3];          // raw inputs, dtype [B][N][C]
  const float* dy[3];        // gradients of the conv outputs, fp32 [B][N][C]
  void* dx[3];               // dtype [B][N][C]
  const float* w_text;       // [3][C][text_k]
  const float* w_vis;        // [3][C][27]
  float* dw_text;            // [3][C][text_k], accumulated
  float* dw_vis;             // [3][C][27], accumulated
  int64_t N, L;
  int B, C, text_k, T, Hg, Wg, pt;
};

// Both conv backward kernels: a CTA covers CB_TOK tokens of one batch item and 32 channels of
// one tensor (one per lane; 8 warps split the tokens), the channel's taps in registers.
constexpr int CB_TOK = 256;

struct TokenPos {   // visual token n >= L of a batch item: its grid position
  int tt, hh, ww;
};
__device__ __forceinline__ TokenPos grid_pos(const ConvBwdArgs& a, int64_t n) {
  const int p = (int)(n - a.L), hw = a.Hg * a.Wg;
  TokenPos t;
  t.tt = p / hw;
  const int rem = p - t.tt * hw;
  t.hh = rem / a.Wg;
  t.ww = rem - t.hh * a.Wg;
  return t;
}

// dx = every output that read x, times its tap weight (the transpose of the conv)
template <typename T>
__global__ void __launch_bounds__(256) conv_bwd_dx_kernel(ConvBwdArgs a) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, tensor = blockIdx.z;
  const int c = blockIdx.y * 32 + lane;
  const int64_t bpi = (a.N + CB_TOK - 1) / CB_TOK;
  const int64_t b = blockIdx.x / bpi, n0 = (blockIdx.x % bpi) * CB_TOK;
  float wv[27], wt[8];
#pragma unroll
  for (int i = 0; i < 27; ++i) wv[i] = a.w_vis[((int64_t)tensor * a.C + c) * 27 + i];
#pragma unroll
  for (int i = 0; i < 8; ++i) wt[i] = i < a.text_k ? a.w_text[((int64_t)tensor * a.C + c) * a.text_k + i] : 0.f;
  const float* dy = (tensor == 0 ? a.dy[0] : tensor == 1 ? a.dy[1] : a.dy[2]) + b * a.N * a.C + c;
  T* dx = static_cast<T*>(tensor == 0 ? a.dx[0] : tensor == 1 ? a.dx[1] : a.dx[2]) + b * a.N * a.C + c;
  const int64_t wc = (int64_t)a.Wg * a.C, hwc = wc * a.Hg;   // one grid row, one frame
  const int64_t n1 = min(n0 + CB_TOK, a.N);
  for (int64_t n = n0 + warp; n < n1; n += 8) {
    float acc = 0.f;
    if (n < a.L) {
      // y[m] reads x[m - (K-1) + j]: x[n] feeds the text outputs m = n + K-1-j < L
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int64_t m = n + (a.text_k - 1) - j;
        if (j < a.text_k && m < a.L) acc += wt[j] * dy[m * a.C];
      }
    } else {
      // the output at (tt - ta + pt, hh - tb + 1, ww - te + 1) reads this token through tap (ta, tb, te);
      // its address is this token's plus fixed per-axis offsets
      const TokenPos t = grid_pos(a, n);
      const float* p = dy + n * a.C;
#pragma unroll
      for (int ta = 0; ta < 3; ++ta) {
        const int t2 = t.tt - ta + a.pt;
        if (t2 < 0 || t2 >= a.T) continue;
        const float* pa = p + (int64_t)(a.pt - ta) * hwc;
#pragma unroll
        for (int tb = 0; tb < 3; ++tb) {
          const int h2 = t.hh - tb + 1;
          if (h2 < 0 || h2 >= a.Hg) continue;
          const float* pb = pa + (int64_t)(1 - tb) * wc;
#pragma unroll
          for (int te = 0; te < 3; ++te) {
            const int w2 = t.ww - te + 1;
            if (w2 >= 0 && w2 < a.Wg) acc += wv[(ta * 3 + tb) * 3 + te] * pb[(1 - te) * a.C];
          }
        }
      }
    }
    dx[n * a.C] = from_f32<T>(acc);
  }
}

// dw = sum over tokens of x * dy per channel and tap: per-warp sums meet in shared memory, then
// one atomic add per (channel, tap) and CTA
template <typename TIn>
__global__ void __launch_bounds__(256) conv_bwd_dw_kernel(ConvBwdArgs a) {
  __shared__ float part[8][35][32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, tensor = blockIdx.z;
  const int c = blockIdx.y * 32 + lane;
  const int64_t bpi = (a.N + CB_TOK - 1) / CB_TOK;
  const int64_t b = blockIdx.x / bpi, n0 = (blockIdx.x % bpi) * CB_TOK;
  const TIn* x = static_cast<const TIn*>(tensor == 0 ? a.x[0] : tensor == 1 ? a.x[1] : a.x[2]) + b * a.N * a.C + c;
  const float* dy = (tensor == 0 ? a.dy[0] : tensor == 1 ? a.dy[1] : a.dy[2]) + b * a.N * a.C + c;
  const int64_t wc = (int64_t)a.Wg * a.C, hwc = wc * a.Hg;   // one grid row, one frame
  float av[27], at[8];
#pragma unroll
  for (int i = 0; i < 27; ++i) av[i] = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) at[i] = 0.f;
  const int64_t n1 = min(n0 + CB_TOK, a.N);
  for (int64_t n = n0 + warp; n < n1; n += 8) {
    const float gv = dy[n * a.C];
    if (n < a.L) {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int64_t s = n - (a.text_k - 1) + j;
        if (j < a.text_k && s >= 0) at[j] += to_f32(x[s * a.C]) * gv;
      }
    } else {
      // tap (ta, tb, te) of this output read x at (tt + ta - pt, hh + tb - 1, ww + te - 1)
      const TokenPos t = grid_pos(a, n);
      const TIn* p = x + n * a.C;
#pragma unroll
      for (int ta = 0; ta < 3; ++ta) {
        const int t2 = t.tt + ta - a.pt;
        if (t2 < 0 || t2 >= a.T) continue;
        const TIn* pa = p + (int64_t)(ta - a.pt) * hwc;
#pragma unroll
        for (int tb = 0; tb < 3; ++tb) {
          const int h2 = t.hh + tb - 1;
          if (h2 < 0 || h2 >= a.Hg) continue;
          const TIn* pb = pa + (int64_t)(tb - 1) * wc;
#pragma unroll
          for (int te = 0; te < 3; ++te) {
            const int w2 = t.ww + te - 1;
            if (w2 >= 0 && w2 < a.Wg) av[(ta * 3 + tb) * 3 + te] += to_f32(pb[(te - 1) * a.C]) * gv;
          }
        }
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 27; ++i) part[warp][i][lane] = av[i];
#pragma unroll
  for (int i = 0; i < 8; ++i) part[warp][27 + i][lane] = at[i];
  __syncthreads();
  for (int e = threadIdx.x; e < 35 * 32; e += 256) {
    const int i = e / 32, l = e % 32;
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) s += part[w][i][l];
    const int cc = blockIdx.y * 32 + l;
    if (i < 27) atomicAdd(a.dw_vis + ((int64_t)tensor * a.C + cc) * 27 + i, s);
    else if (i - 27 < a.text_k) atomicAdd(a.dw_text + ((int64_t)tensor * a.C + cc) * a.text_k + (i - 27), s);
  }
}

struct BwdLayout {
  size_t act32, dbeta, ckpt, total;
  int n_ck;
};

BwdLayout bwd_layout(const Dims& d) {
  BwdLayout l;
  const size_t elems = (size_t)d.B * d.N * d.H * d.dk;
  l.act32 = align256(elems * sizeof(float));
  l.dbeta = align256((size_t)d.B * d.N * d.H * sizeof(float));
  l.n_ck = (int)((d.N + KC - 1) / KC);
  l.ckpt = align256((size_t)d.B * d.H * l.n_ck * d.dk * d.dk * sizeof(float));
  l.total = 256 + 6 * l.act32 + l.dbeta + l.ckpt;
  return l;
}

template <int DK>
cudaError_t launch_scan_bwd(const ScanBwdArgs& a, const Dims& d, cudaStream_t s) {
  const dim3 grid((unsigned)(DK / CWB), (unsigned)d.H, (unsigned)d.B);
  bwd_states_kernel<DK><<<grid, DK, 0, s>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  constexpr size_t smem = scan_bwd_smem<DK>();
  if ((e = cudaFuncSetAttribute(bwd_scan_kernel<DK>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) !=
      cudaSuccess)
    return e;
  bwd_scan_kernel<DK><<<grid, 2 * DK, smem, s>>>(a);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_conv_bwd(const ConvBwdArgs& c, const Dims& d, cudaStream_t s) {
  const dim3 grid((unsigned)(d.B * ((d.N + CB_TOK - 1) / CB_TOK)), (unsigned)(c.C / 32), 3);
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
  float* ckpt = reinterpret_cast<float*>(base + 6 * l.act32 + l.dbeta);
  const int C = d.H * d.dk;
  const size_t elems = (size_t)d.B * d.N * d.H * d.dk;
  cudaError_t e;
  if ((e = cudaMemsetAsync(dw_text, 0, sizeof(float) * 3 * C * d.text_k, s)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(dw_vis, 0, sizeof(float) * 3 * C * 27, s)) != cudaSuccess) return e;
  if (d.N == 0) {
    if (!dS0) return cudaSuccess;
    const size_t bytes = (size_t)d.B * d.H * d.dk * d.dv * sizeof(float);
    return dSN ? cudaMemcpyAsync(dS0, dSN, bytes, cudaMemcpyDeviceToDevice, s) : cudaMemsetAsync(dS0, 0, bytes, s);
  }
  for (int i = 3; i < 5; ++i)
    if ((e = cudaMemsetAsync(act[i], 0, elems * sizeof(float), s)) != cudaSuccess) return e;   // dq', dk'
  if ((e = cudaMemsetAsync(dla, 0, elems * sizeof(float), s)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(dbeta32, 0, (size_t)d.B * d.N * d.H * sizeof(float), s)) != cudaSuccess) return e;
  // 1. the convolved activations, fp32
  if ((e = launch_shortconv(d, dt, q, k, v, w_text, w_vis, act[0], act[1], act[2], s, launches, false, true)) !=
      cudaSuccess)
    return e;
  // 2. scan backward
  ScanBwdArgs a{act[0], act[1], act[2], log_alpha, beta, S0, d_o, dSN, ckpt, act[3], act[4], act[5], dla, dbeta32,
                dS0, d.N, d.H, l.n_ck, dt == KDA_DT_BF16};
  e = d.dk == 128 ? launch_scan_bwd<128>(a, d, s) : launch_scan_bwd<64>(a, d, s);
  if (e != cudaSuccess) return e;
  const int64_t nb = (int64_t)d.B * d.N * d.H;
  if (dt == KDA_DT_BF16)
    bwd_beta_kernel<__nv_bfloat16><<<(unsigned)((nb + 255) / 256), 256, 0, s>>>(dbeta32, static_cast<__nv_bfloat16*>(dbeta), nb);
  else
    bwd_beta_kernel<float><<<(unsigned)((nb + 255) / 256), 256, 0, s>>>(dbeta32, static_cast<float*>(dbeta), nb);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // 3. conv backward
  ConvBwdArgs c;
  c.x[0] = q; c.x[1] = k; c.x[2] = v;
  c.dy[0] = act[3]; c.dy[1] = act[4]; c.dy[2] = act[5];
  c.dx[0] = dq; c.dx[1] = dk; c.dx[2] = dv;
  c.w_text = w_text; c.w_vis = w_vis; c.dw_text = dw_text; c.dw_vis = dw_vis;
  c.N = d.N; c.L = d.L; c.B = d.B; c.C = C; c.text_k = d.text_k; c.T = d.T; c.Hg = d.Hg; c.Wg = d.Wg; c.pt = d.pt;
  e = dt == KDA_DT_BF16 ? launch_conv_bwd<__nv_bfloat16>(c, d, s) : launch_conv_bwd<float>(c, d, s);
  if (e != cudaSuccess) return e;
  if (launches) *launches += 2 + 1 + 2;
  return cudaSuccess;
}

}  // namespace kda
