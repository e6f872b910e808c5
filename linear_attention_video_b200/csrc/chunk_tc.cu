// Chunked KDA scan on the sm_100a tensor cores (tcgen05, fp16 operands, fp32
// accumulation in TMEM), for d_k = d_v = 128.
//
// Recurrence (paper.rainbus.top, section 方法步骤详情 step (5)), per head:
//   S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,   o_t = S_t^T q_t.
//
// The sequence is cut into blocks of 128 tokens, each made of two 64-token
// sub-chunks.  For a sub-chunk with g_r = sum_{i<=r} log alpha_i (per key
// channel, from the sub-chunk start), a reference g_m = g_31 (mid point) keeps
// every exponential factor within e^{+-9} so fp16 operands cannot overflow:
//   KG = K e^{g-g_m},  QG = Q e^{g-g_m},  KN = K e^{g_m-g}
//   A  = strict_lower(Diag(beta) KG KN^T),  P = lower(QG KN^T)
//   T  = (I + A)^{-1} Diag(beta),  W' = T KG,  U~ = T V
//   K~ = KN e^{g_l-g_m}  (g_l = last g),   Gamma = e^{g_l}
//   M_s = Diag(Gamma) - (K~^T W') Diag(e^{g_m}),   B_s = K~^T U~
//   Q^_s = (QG - P W') Diag(e^{g_m}),   O'_s = P U~
// so that, entering with state S, the sub-chunk gives O = Q^_s S + O'_s and
// leaves S <- M_s S + B_s.  Two sub-chunks compose into one 128-token block:
//   M = M_2 M_1,  B = M_2 B_1 + B_2,  R = [Q^_1 ; Q^_2 M_1],  O'' = [O'_1 ; Q^_2 B_1 + O'_2]
// and the block maps S to O = R S + O'' and S <- M S + B.
//
// Three kernels:
//   kda_tc_prep   one CTA per (batch item, head, block): everything above,
//                 written to the workspace (M, B, R, O'' per block).
//   kda_tc_chain  one CTA per (batch item, head, half of the value columns):
//                 the serial pass S <- M S + B, state kept in registers (fp32),
//                 saving the state entering each block.
//   kda_tc_out    one CTA per (batch item, head, block): O = R S + O''.
// Padding tokens of the last block carry k = q = v = 0, beta = 0, log alpha = 0.
#include "common.cuh"
#include "tc.cuh"

#include <cuda_fp16.h>

namespace kda {
namespace {

using namespace tc;

constexpr int BLK = 128;          // tokens per block (one serial step)
constexpr int SUB = 64;           // tokens per sub-chunk
constexpr int D = 128;            // d_k = d_v
constexpr float kRange = 9.f;     // max |g - g_m| allowed for the fp16 factors

// Workspace bytes per (batch item, head, block).
constexpr size_t kMBytes = 32768;   // M: fp16, 2 K-major panels [128][64]
constexpr size_t kBBytes = 65536;   // B: fp32, [half][c/4][a][4]
constexpr size_t kRBytes = 32768;   // R: fp16, 2 K-major panels [128][64]
constexpr size_t kOBytes = 65536;   // O'': fp32, float4 units [c/4][r]
constexpr size_t kSBytes = 32768;   // S entering the block: fp16, 2 MN-major panels [128][64]
constexpr size_t kBlockBytes = kMBytes + kBBytes + kRBytes + kOBytes + kSBytes;

// ---------------------------------------------------------------------------
// small helpers
// ---------------------------------------------------------------------------

__device__ __forceinline__ float2 ld_act2(const __half* p) { return __half22float2(*reinterpret_cast<const __half2*>(p)); }
__device__ __forceinline__ float2 ld_act2(const __nv_bfloat16* p) {
  return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
}

__device__ __forceinline__ void st_h2(uint8_t* p, float a, float b) {
  *reinterpret_cast<__half2*>(p) = __floats2half2_rn(a, b);
}

// 16 consecutive fp32 values -> 16 fp16 at (row, col0..col0+15) of a swizzled panel.
__device__ __forceinline__ void st_row16_h(uint8_t* panel, int row, int col0, const float (&v)[16]) {
  uint32_t w[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    __half2 h = __floats2half2_rn(v[2 * i], v[2 * i + 1]);
    w[i] = *reinterpret_cast<uint32_t*>(&h);
  }
  *reinterpret_cast<uint4*>(panel + swz_off(row, col0)) = make_uint4(w[0], w[1], w[2], w[3]);
  *reinterpret_cast<uint4*>(panel + swz_off(row, col0 + 8)) = make_uint4(w[4], w[5], w[6], w[7]);
}

// 16 fp16 at (row, col0..) of a swizzled panel -> fp32
__device__ __forceinline__ void ld_row16_h(const uint8_t* panel, int row, int col0, float (&v)[16]) {
  const uint4 a = *reinterpret_cast<const uint4*>(panel + swz_off(row, col0));
  const uint4 b = *reinterpret_cast<const uint4*>(panel + swz_off(row, col0 + 8));
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const __half2 h = *reinterpret_cast<const __half2*>(&w[i]);
    const float2 f = __half22float2(h);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}

__device__ __forceinline__ uint32_t tmem_at(uint32_t base, int lane0, int col) {
  return base + ((uint32_t)lane0 << 16) + (uint32_t)col;
}

// Waits on the MMA barrier; on timeout records the status.  Returns false on timeout.
__device__ __forceinline__ bool wait_mma(uint64_t* bar, uint32_t& phase, uint32_t* status, bool alive) {
  if (!alive) return false;   // nothing was issued
  const bool ok = mbar_wait(bar, phase);
  phase ^= 1u;
  if (!ok) set_status(status, KDA_ERR_TIMEOUT);
  return ok;
}

// ---------------------------------------------------------------------------
// kda_tc_prep
// ---------------------------------------------------------------------------
// shared memory map (bytes from a 1024-aligned base)
constexpr uint32_t OFF_KQ = 0;          // [128 rows][128] fp16: rows 0-63 KG (later W'), 64-127 QG; 2 panels of 16 KB
constexpr uint32_t OFF_KN = 32768;      // [64][128] fp16: KN, then K~; 2 panels of 8 KB
constexpr uint32_t OFF_VV = 49152;      // [64][128] fp16: V, then U~ (then Q^_2); 2 panels of 8 KB
constexpr uint32_t OFF_TT = 65536;      // [64][64] fp16: T
constexpr uint32_t OFF_PP = 73728;      // [64][64] fp16: P
constexpr uint32_t OFF_M1 = 81920;      // [128][128] fp16: M_1; 2 panels of 16 KB
constexpr uint32_t OFF_B1 = 114688;     // [128][128] fp16: B_1; 2 panels of 16 KB
constexpr uint32_t OFF_AS = 147456;     // fp32 [64][65]: A (strictly lower, beta applied)
constexpr uint32_t OFF_XS = 164096;     // fp32 [64][65]: (I + A)^{-1}
constexpr uint32_t OFF_YS = 180736;     // fp32 [32][33]: merge scratch
constexpr uint32_t OFF_MISC = 184960;   // beta[64], egm[128], egl[128], ekt[128], gm[128], tot[128], bars, tmem
constexpr uint32_t PREP_SMEM = OFF_MISC + 4096 + 1024;   // + alignment slack

constexpr int LDX = 65;

// TMEM columns
constexpr int C_AP = 0, C_W = 64, C_U = 192;
constexpr int C_MK = 0, C_BK = 128, C_PW = 256, C_PU = 384;

struct PrepArgs {
  const void* q; const void* k; const void* v;
  const float* la; const void* beta;
  uint8_t* ws;            // block records
  int64_t N; int H; int n_blocks;
  uint32_t* status;
};

// Blocked inverse of the unit lower-triangular (I + A), A in As (strictly lower).
__device__ void unit_lower_inverse64(const float* As, float* Xs, float* Ys) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // diagonal 16x16 blocks: warp b, lane l = column 16b + l
  if (warp < 4 && lane < 16) {
    const int b = warp, l = lane, o = 16 * b;
    float x[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) {
      float acc = 0.f;
#pragma unroll
      for (int m = 0; m < r; ++m) acc += As[(o + r) * LDX + o + m] * x[m];
      x[r] = r < l ? 0.f : (r == l ? 1.f : -acc);
    }
#pragma unroll
    for (int r = 0; r < 16; ++r) Xs[(o + r) * LDX + o + l] = x[r];
  }
  __syncthreads();
  // 32x32 merges: for p in {0,1}: X[32p+16.., 32p..] = -X22 (A21 X11); one 2x1 tile per thread
  {
    const int p = tid >> 7, e = tid & 127;
    const int o = 32 * p;
    float* Y = Ys + p * 16 * 17;
    const int r0 = 2 * (e >> 4), c = e & 15;
    {
      float a0 = 0.f, a1 = 0.f;
      for (int m = c; m < 16; ++m) {
        const float x = Xs[(o + m) * LDX + o + c];
        a0 += As[(o + 16 + r0) * LDX + o + m] * x;
        a1 += As[(o + 17 + r0) * LDX + o + m] * x;
      }
      Y[r0 * 17 + c] = a0;
      Y[(r0 + 1) * 17 + c] = a1;
    }
    __syncthreads();
    {
      float a0 = 0.f, a1 = 0.f;
      for (int m = 0; m <= r0 + 1; ++m) {
        const float y = Y[m * 17 + c];
        a0 += (m <= r0 ? Xs[(o + 16 + r0) * LDX + o + 16 + m] : 0.f) * y;
        a1 += Xs[(o + 17 + r0) * LDX + o + 16 + m] * y;
      }
      Xs[(o + 16 + r0) * LDX + o + c] = -a0;
      Xs[(o + 17 + r0) * LDX + o + c] = -a1;
    }
    __syncthreads();
  }
  // 64 merge: X[32.., 0..31] = -X22 (A21 X11); one 2x2 tile per thread
  {
    const int r0 = 2 * (tid >> 4), c0 = 2 * (tid & 15);
    float a00 = 0.f, a01 = 0.f, a10 = 0.f, a11 = 0.f;
    for (int m = c0; m < 32; ++m) {
      const float x0 = Xs[m * LDX + c0], x1 = Xs[m * LDX + c0 + 1];
      const float u0 = As[(32 + r0) * LDX + m], u1 = As[(33 + r0) * LDX + m];
      a00 += u0 * x0; a01 += u0 * x1; a10 += u1 * x0; a11 += u1 * x1;
    }
    Ys[r0 * 33 + c0] = a00; Ys[r0 * 33 + c0 + 1] = a01;
    Ys[(r0 + 1) * 33 + c0] = a10; Ys[(r0 + 1) * 33 + c0 + 1] = a11;
    __syncthreads();
    a00 = a01 = a10 = a11 = 0.f;
    for (int m = 0; m <= r0 + 1; ++m) {
      const float y0 = Ys[m * 33 + c0], y1 = Ys[m * 33 + c0 + 1];
      const float u0 = m <= r0 ? Xs[(32 + r0) * LDX + 32 + m] : 0.f, u1 = Xs[(33 + r0) * LDX + 32 + m];
      a00 += u0 * y0; a01 += u0 * y1; a10 += u1 * y0; a11 += u1 * y1;
    }
    Xs[(32 + r0) * LDX + c0] = -a00; Xs[(32 + r0) * LDX + c0 + 1] = -a01;
    Xs[(33 + r0) * LDX + c0] = -a10; Xs[(33 + r0) * LDX + c0 + 1] = -a11;
    __syncthreads();
  }
}

template <typename TIn>
__global__ void __launch_bounds__(256, 1) kda_tc_prep(PrepArgs a) {
  extern __shared__ uint8_t dyn[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dyn) + 1023) & ~uintptr_t(1023));
  uint8_t* KQ = sm + OFF_KQ;
  uint8_t* KN = sm + OFF_KN;
  uint8_t* VV = sm + OFF_VV;
  uint8_t* TT = sm + OFF_TT;
  uint8_t* PP = sm + OFF_PP;
  uint8_t* M1 = sm + OFF_M1;
  uint8_t* B1 = sm + OFF_B1;
  float* As = reinterpret_cast<float*>(sm + OFF_AS);
  float* Xs = reinterpret_cast<float*>(sm + OFF_XS);
  float* Ys = reinterpret_cast<float*>(sm + OFF_YS);
  float* beta_s = reinterpret_cast<float*>(sm + OFF_MISC);     // 64
  float* egm = beta_s + 64;                                     // 128: e^{g_m}
  float* egl = egm + 128;                                       // 128: e^{g_l}
  float* ekt = egl + 128;                                       // 128: e^{g_l - g_m}
  float* gm_s = ekt + 128;                                      // 128
  float* tot_s = gm_s + 128;                                    // 128
  uint64_t* bar = reinterpret_cast<uint64_t*>(tot_s + 128);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 2);
  int* range_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int blk = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int64_t tok_stride = (int64_t)a.H * D;
  const TIn* qb = static_cast<const TIn*>(a.q) + (int64_t)b * a.N * tok_stride + (int64_t)h * D;
  const TIn* kb = static_cast<const TIn*>(a.k) + (int64_t)b * a.N * tok_stride + (int64_t)h * D;
  const TIn* vb = static_cast<const TIn*>(a.v) + (int64_t)b * a.N * tok_stride + (int64_t)h * D;
  const float* lab = a.la + (int64_t)b * a.N * tok_stride + (int64_t)h * D;
  const __nv_bfloat16* bb = static_cast<const __nv_bfloat16*>(a.beta) + (int64_t)b * a.N * a.H + h;
  uint8_t* rec = a.ws + (((int64_t)b * a.H + h) * a.n_blocks + blk) * kBlockBytes;
  uint8_t* gM = rec;
  float* gB = reinterpret_cast<float*>(rec + kMBytes);
  uint8_t* gR = rec + kMBytes + kBBytes;
  float* gO = reinterpret_cast<float*>(rec + kMBytes + kBBytes + kRBytes);

  if (*(volatile uint32_t*)a.status == KDA_ERR_TIMEOUT) return;   // an earlier CTA gave up: skip the work
  if (warp == 0) { tmem_alloc(tmem_slot, 512); tmem_relinquish(); }
  if (tid == 0) { mbar_init(bar, 1); fence_mbar_init(); *range_flag = 0; }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tm = *tmem_slot;
  uint32_t phase = 0;
  bool alive = true;

  const uint32_t id_ap = idesc_f16(128, 64, false, false);
  const uint32_t id_64x128_kmn = idesc_f16(64, 128, false, true);
  const uint32_t id_128x128_mnmn = idesc_f16(128, 128, true, true);
  const uint32_t id_128x128_kmn = idesc_f16(128, 128, false, true);

  for (int s = 0; s < 2; ++s) {
    const int64_t t0 = (int64_t)blk * BLK + s * SUB;
    const int nv = (int)max((int64_t)0, min((int64_t)SUB, a.N - t0));
    // ---------------- load + gate factors ----------------
    // raw k, q, v rows (256 B each) -> staging with 16-byte asynchronous copies
    // spread over all threads; staging lives in the solve scratch and T/P
    // tiles, which are dead at this point
    uint8_t* stg_k = sm + OFF_AS;
    uint8_t* stg_q = sm + OFF_AS + 16384;
    uint8_t* stg_v = sm + OFF_TT;
    for (int e = tid; e < nv * 16; e += 256) {
      const int r = e >> 4, ch = (e & 15) * 8;     // row, first of 8 channels
      const int64_t go = (t0 + r) * tok_stride + ch;
      cp_async16(stg_k + r * 256 + ch * 2, kb + go);
      cp_async16(stg_q + r * 256 + ch * 2, qb + go);
      cp_async16(stg_v + r * 256 + ch * 2, vb + go);
    }
    cp_async_commit();
    {
      // thread: channels 2cp, 2cp+1 and tokens 16*qt .. 16*qt+15 of the sub-chunk
      const int cp = (tid & 31) + 32 * ((tid >> 5) & 1);
      const int qt = tid >> 6;
      const int c = 2 * cp;
      float2 gl[16];
#pragma unroll
      for (int t = 0; t < 16; ++t) {
        const int tok = 16 * qt + t;
        gl[t] = tok < nv ? *reinterpret_cast<const float2*>(lab + (t0 + tok) * tok_stride + c) : make_float2(0.f, 0.f);
      }
#pragma unroll
      for (int t = 1; t < 16; ++t) { gl[t].x += gl[t - 1].x; gl[t].y += gl[t - 1].y; }
      float2* qtot = reinterpret_cast<float2*>(Ys);      // [4][64] quarter totals (Ys is free here)
      qtot[qt * 64 + cp] = gl[15];
      if (tid < SUB) beta_s[tid] = tid < nv ? __bfloat162float(bb[(t0 + tid) * a.H]) : 0.f;
      __syncthreads();
      float2 pre = make_float2(0.f, 0.f), gmv = make_float2(0.f, 0.f), tot = make_float2(0.f, 0.f);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 v = qtot[j * 64 + cp];
        if (j < qt) { pre.x += v.x; pre.y += v.y; }
        if (j < 2) { gmv.x += v.x; gmv.y += v.y; } else { tot.x += v.x; tot.y += v.y; }
      }
      if (qt == 0) {
        gm_s[c] = gmv.x; gm_s[c + 1] = gmv.y;       // g_m: decay through token 31
        tot_s[c] = tot.x; tot_s[c + 1] = tot.y;     // decay over tokens 32..63
      }
      // exponent x = g - g_m; the extremes sit at token 0 and token 63
      if (qt == 0 && (pre.x + gl[0].x - gmv.x > kRange || pre.y + gl[0].y - gmv.y > kRange)) *range_flag = 1;
      if (qt == 3 && (-tot.x > kRange || -tot.y > kRange)) *range_flag = 1;
      cp_async_wait_all();
      __syncthreads();
      const bool got = true;
      const int pnl = c >> 6, cc = c & 63;
      uint8_t* kq = KQ + pnl * 16384;
      uint8_t* kn = KN + pnl * 8192;
      uint8_t* vv = VV + pnl * 8192;
#pragma unroll 4
      for (int t = 0; t < 16; ++t) {
        const int tok = 16 * qt + t;
        float2 kv = make_float2(0.f, 0.f), qv = kv, vv2 = kv;
        if (tok < nv && got) {
          kv = ld_act2(reinterpret_cast<const TIn*>(stg_k + tok * 256) + c);
          qv = ld_act2(reinterpret_cast<const TIn*>(stg_q + tok * 256) + c);
          vv2 = ld_act2(reinterpret_cast<const TIn*>(stg_v + tok * 256) + c);
        }
        const float x0 = pre.x + gl[t].x - gmv.x, x1 = pre.y + gl[t].y - gmv.y;
        const float ep0 = __expf(x0), ep1 = __expf(x1), en0 = __expf(-x0), en1 = __expf(-x1);
        const uint32_t off = swz_off(tok, cc);
        st_h2(kq + off, kv.x * ep0, kv.y * ep1);
        st_h2(kq + swz_off(64 + tok, cc), qv.x * ep0, qv.y * ep1);
        st_h2(kn + off, kv.x * en0, kv.y * en1);
        st_h2(vv + off, vv2.x, vv2.y);
      }
    }
    fence_proxy_async();
    __syncthreads();
    if (tid < 128) {
      const float gm = gm_s[tid], tot = tot_s[tid];
      egm[tid] = __expf(gm);
      egl[tid] = __expf(gm + tot);
      ekt[tid] = __expf(tot);
    }
    // ---------------- A, P = [KG; QG] KN^T ----------------
    if (tid == 0 && alive) {
      fence_after_sync();
      for (int k16 = 0; k16 < 8; ++k16)
        mma_ss(tmem_at(tm, 0, C_AP), desc_kmajor(smem_u32(KQ), k16, 16384), desc_kmajor(smem_u32(KN), k16, 8192),
               id_ap, k16 > 0);
      mma_commit(bar);
    }
    alive = __syncthreads_and(wait_mma(bar, phase, a.status, alive));
    fence_after_sync();
    {
      // A rows (TMEM lanes 0-63) -> As (beta, strict lower); P rows (lanes 64-127) -> PP (lower)
      const int sub = warp & 3, chalf = warp >> 2;
      const int row = 32 * sub + lane;
      for (int cb = 0; cb < 2; ++cb) {
        const int col0 = 32 * chalf + 16 * cb;
        float v[16];
        tmem_ld16(tmem_at(tm, 32 * sub, C_AP + col0), v);
        tmem_wait_ld();
        if (sub < 2) {
          const float bt = beta_s[row];
#pragma unroll
          for (int j = 0; j < 16; ++j) As[row * LDX + col0 + j] = (col0 + j < row) ? bt * v[j] : 0.f;
        } else {
          const int r = row - 64;
#pragma unroll
          for (int j = 0; j < 16; ++j) v[j] = (col0 + j <= r) ? v[j] : 0.f;
          st_row16_h(PP, r, col0, v);
        }
      }
    }
    for (int i = tid; i < SUB * LDX; i += 256) Xs[i] = 0.f;
    fence_before_sync();
    __syncthreads();
    unit_lower_inverse64(As, Xs, Ys);
    // T = X Diag(beta) -> TT (fp16, [r][i])
    for (int e = tid; e < SUB * 8; e += 256) {
      const int r = e >> 3, c0 = (e & 7) * 8;
      float v[16];
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = Xs[r * LDX + c0 + j] * beta_s[c0 + j];
      uint32_t w[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        __half2 hh = __floats2half2_rn(v[2 * j], v[2 * j + 1]);
        w[j] = *reinterpret_cast<uint32_t*>(&hh);
      }
      *reinterpret_cast<uint4*>(TT + swz_off(r, c0)) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    fence_proxy_async();
    __syncthreads();
    // ---------------- W' = T KG, U~ = T V ----------------
    if (tid == 0 && alive) {
      fence_after_sync();
      for (int k16 = 0; k16 < 4; ++k16) {
        const uint64_t ad = desc_kmajor(smem_u32(TT), k16, 8192);
        mma_ss(tmem_at(tm, 0, C_W), ad, desc_mnmajor(smem_u32(KQ), k16, 16384), id_64x128_kmn, k16 > 0);
        mma_ss(tmem_at(tm, 0, C_U), ad, desc_mnmajor(smem_u32(VV), k16, 8192), id_64x128_kmn, k16 > 0);
      }
      mma_commit(bar);
    }
    // KN -> K~ = KN e^{g_l - g_m} in place (KN is no longer read by the tensor core)
    for (int e = tid; e < SUB * 16; e += 256) {
      const int r = e >> 4, ch = (e & 15) * 8;           // row, first of 8 channels
      uint8_t* pnl = KN + (ch >> 6) * 8192;
      uint4* p = reinterpret_cast<uint4*>(pnl + swz_off(r, ch & 63));
      uint4 u = *p;
      uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float2 f = __half22float2(*reinterpret_cast<__half2*>(&w[j]));
        f.x *= ekt[ch + 2 * j];
        f.y *= ekt[ch + 2 * j + 1];
        __half2 hh = __floats2half2_rn(f.x, f.y);
        w[j] = *reinterpret_cast<uint32_t*>(&hh);
      }
      *p = make_uint4(w[0], w[1], w[2], w[3]);
    }
    fence_proxy_async();
    alive = __syncthreads_and(wait_mma(bar, phase, a.status, alive));
    fence_after_sync();
    // W' -> KQ rows 0-63 (fp16), U~ -> VV (fp16); M=64 accumulator layout
    {
      const int sub = warp & 3, chalf = warp >> 2;
      const int row = 16 * sub + lane;     // valid for lane < 16
      for (int cb = 0; cb < 4; ++cb) {
        const int col0 = 64 * chalf + 16 * cb;
        float w[16], u[16];
        tmem_ld16(tmem_at(tm, 32 * sub, C_W + col0), w);
        tmem_ld16(tmem_at(tm, 32 * sub, C_U + col0), u);
        tmem_wait_ld();
        if (lane < 16) {
          st_row16_h(KQ + (col0 >> 6) * 16384, row, col0 & 63, w);
          st_row16_h(VV + (col0 >> 6) * 8192, row, col0 & 63, u);
        }
      }
    }
    fence_proxy_async();
    fence_before_sync();
    __syncthreads();
    // ---------------- K~^T W', K~^T U~, P W', P U~ ----------------
    if (tid == 0 && alive) {
      fence_after_sync();
      for (int k16 = 0; k16 < 4; ++k16) {
        const uint64_t kt = desc_mnmajor(smem_u32(KN), k16, 8192);
        const uint64_t wd = desc_mnmajor(smem_u32(KQ), k16, 16384);
        const uint64_t ud = desc_mnmajor(smem_u32(VV), k16, 8192);
        const uint64_t pd = desc_kmajor(smem_u32(PP), k16, 8192);
        mma_ss(tmem_at(tm, 0, C_MK), kt, wd, id_128x128_mnmn, k16 > 0);
        mma_ss(tmem_at(tm, 0, C_BK), kt, ud, id_128x128_mnmn, k16 > 0);
        mma_ss(tmem_at(tm, 0, C_PW), pd, wd, id_64x128_kmn, k16 > 0);
        mma_ss(tmem_at(tm, 0, C_PU), pd, ud, id_64x128_kmn, k16 > 0);
      }
      mma_commit(bar);
    }
    alive = __syncthreads_and(wait_mma(bar, phase, a.status, alive));
    fence_after_sync();
    const int sub = warp & 3, chalf = warp >> 2;
    if (s == 0) {
      // M_1 = Diag(e^{g_l}) - MK Diag(e^{g_m}) -> M1 tile;  B_1 -> B1 tile
      const int row = 32 * sub + lane;
      for (int cb = 0; cb < 4; ++cb) {
        const int col0 = 64 * chalf + 16 * cb;
        float m[16], bv[16];
        tmem_ld16(tmem_at(tm, 32 * sub, C_MK + col0), m);
        tmem_ld16(tmem_at(tm, 32 * sub, C_BK + col0), bv);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j) m[j] = (row == col0 + j ? egl[row] : 0.f) - m[j] * egm[col0 + j];
        st_row16_h(M1 + (col0 >> 6) * 16384, row, col0 & 63, m);
        st_row16_h(B1 + (col0 >> 6) * 16384, row, col0 & 63, bv);
      }
      // R_1 = (QG - P W') Diag(e^{g_m}) -> global R rows 0-63;  O'_1 -> global O'' rows 0-63
      const int r = 16 * sub + lane;
      for (int cb = 0; cb < 4; ++cb) {
        const int col0 = 64 * chalf + 16 * cb;
        float pw[16], pu[16];
        tmem_ld16(tmem_at(tm, 32 * sub, C_PW + col0), pw);
        tmem_ld16(tmem_at(tm, 32 * sub, C_PU + col0), pu);
        tmem_wait_ld();
        if (lane < 16) {
          float qg[16];
          ld_row16_h(KQ + (col0 >> 6) * 16384, 64 + r, col0 & 63, qg);
#pragma unroll
          for (int j = 0; j < 16; ++j) qg[j] = (qg[j] - pw[j]) * egm[col0 + j];
          st_row16_h(gR + (col0 >> 6) * 16384, r, col0 & 63, qg);
          float4* o4 = reinterpret_cast<float4*>(gO);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            o4[((col0 >> 2) + j) * 128 + r] = make_float4(pu[4 * j], pu[4 * j + 1], pu[4 * j + 2], pu[4 * j + 3]);
        }
      }
      fence_proxy_async();
      fence_before_sync();
      __syncthreads();
    } else {
      // Q^_2 = (QG - P W') Diag(e^{g_m}) -> VV region (U~ no longer needed)
      {
        const int r = 16 * sub + lane;
        for (int cb = 0; cb < 4; ++cb) {
          const int col0 = 64 * chalf + 16 * cb;
          float pw[16];
          tmem_ld16(tmem_at(tm, 32 * sub, C_PW + col0), pw);
          tmem_wait_ld();
          if (lane < 16) {
            float qg[16];
            ld_row16_h(KQ + (col0 >> 6) * 16384, 64 + r, col0 & 63, qg);
#pragma unroll
            for (int j = 0; j < 16; ++j) qg[j] = (qg[j] - pw[j]) * egm[col0 + j];
            st_row16_h(VV + (col0 >> 6) * 8192, r, col0 & 63, qg);
          }
        }
      }
      __syncthreads();
      // M_2 -> KQ region (A operand, K-major, 2 panels of 16 KB)
      {
        const int row = 32 * sub + lane;
        for (int cb = 0; cb < 4; ++cb) {
          const int col0 = 64 * chalf + 16 * cb;
          float m[16];
          tmem_ld16(tmem_at(tm, 32 * sub, C_MK + col0), m);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j) m[j] = (row == col0 + j ? egl[row] : 0.f) - m[j] * egm[col0 + j];
          st_row16_h(KQ + (col0 >> 6) * 16384, row, col0 & 63, m);
        }
      }
      fence_proxy_async();
      fence_before_sync();
      __syncthreads();
      // ---------------- combine ----------------
      if (tid == 0 && alive) {
        fence_after_sync();
        const uint32_t id_q = idesc_f16(64, 128, false, true);
        for (int k16 = 0; k16 < 8; ++k16) {
          const uint64_t m2 = desc_kmajor(smem_u32(KQ), k16, 16384);
          const uint64_t q2 = desc_kmajor(smem_u32(VV), k16, 8192);
          const uint64_t m1 = desc_mnmajor(smem_u32(M1), k16, 16384);
          const uint64_t b1 = desc_mnmajor(smem_u32(B1), k16, 16384);
          mma_ss(tmem_at(tm, 0, C_MK), m2, m1, id_128x128_kmn, k16 > 0);   // M = M_2 M_1
          mma_ss(tmem_at(tm, 0, C_BK), m2, b1, id_128x128_kmn, 1);         // B = B_2 + M_2 B_1
          mma_ss(tmem_at(tm, 0, C_PW), q2, m1, id_q, k16 > 0);             // R_2 = Q^_2 M_1
          mma_ss(tmem_at(tm, 0, C_PU), q2, b1, id_q, 1);                   // O''_2 = O'_2 + Q^_2 B_1
        }
        mma_commit(bar);
      }
      alive = __syncthreads_and(wait_mma(bar, phase, a.status, alive));
      fence_after_sync();
      {
        const int row = 32 * sub + lane;
        for (int cb = 0; cb < 4; ++cb) {
          const int col0 = 64 * chalf + 16 * cb;
          float m[16], bv[16];
          tmem_ld16(tmem_at(tm, 32 * sub, C_MK + col0), m);
          tmem_ld16(tmem_at(tm, 32 * sub, C_BK + col0), bv);
          tmem_wait_ld();
          st_row16_h(gM + (col0 >> 6) * 16384, row, col0 & 63, m);
          // B in [half][c/4][a][4] layout (half = col / 64)
          const int hv = col0 >> 6;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int cq = ((col0 & 63) >> 2) + j;
            reinterpret_cast<float4*>(gB)[((hv * 16 + cq) * 128) + row] =
                make_float4(bv[4 * j], bv[4 * j + 1], bv[4 * j + 2], bv[4 * j + 3]);
          }
        }
        const int r = 16 * sub + lane;
        for (int cb = 0; cb < 4; ++cb) {
          const int col0 = 64 * chalf + 16 * cb;
          float rr[16], oo[16];
          tmem_ld16(tmem_at(tm, 32 * sub, C_PW + col0), rr);
          tmem_ld16(tmem_at(tm, 32 * sub, C_PU + col0), oo);
          tmem_wait_ld();
          if (lane < 16) {
            st_row16_h(gR + (col0 >> 6) * 16384, 64 + r, col0 & 63, rr);
            float4* o4 = reinterpret_cast<float4*>(gO);
#pragma unroll
            for (int j = 0; j < 4; ++j)
              o4[((col0 >> 2) + j) * 128 + 64 + r] =
                  make_float4(oo[4 * j], oo[4 * j + 1], oo[4 * j + 2], oo[4 * j + 3]);
          }
        }
      }
    }
  }
  if (tid == 0 && *range_flag) set_status(a.status, KDA_ERR_RANGE);
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  if (warp == 0) tmem_dealloc(tm, 512);
}

// ---------------------------------------------------------------------------
// kda_tc_chain: S <- M S + B over all blocks, per (b, h, half of value columns)
// ---------------------------------------------------------------------------
constexpr int CH_STAGES = 3;
constexpr uint32_t CH_OFF_S = 0;                         // S fp16 [128][64] MN-major panel (16 KB)
constexpr uint32_t CH_OFF_RING = 16384;                  // stages of {M 32 KB, B-half 32 KB}
constexpr uint32_t CH_STAGE_BYTES = 65536;
constexpr uint32_t CH_OFF_BAR = CH_OFF_RING + CH_STAGES * CH_STAGE_BYTES;
constexpr uint32_t CHAIN_SMEM = CH_OFF_BAR + 256 + 1024;

struct ChainArgs {
  uint8_t* ws;
  const float* S0;
  float* SN;
  int H; int n_blocks;
  uint32_t* status;
};

__global__ void __launch_bounds__(128, 1) kda_tc_chain(ChainArgs a) {
  extern __shared__ uint8_t dyn[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dyn) + 1023) & ~uintptr_t(1023));
  uint8_t* Ssm = sm + CH_OFF_S;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + CH_OFF_BAR);   // [0..2] loads, [3] mma
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 4);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int half = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int64_t rec0 = ((int64_t)b * a.H + h) * a.n_blocks;

  if (warp == 0) { tmem_alloc(tmem_slot, 64); tmem_relinquish(); }
  if (tid == 0) {
    for (int i = 0; i < 4; ++i) mbar_init(&bars[i], 1);
    fence_mbar_init();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tm = *tmem_slot;

  auto issue = [&](int j) {
    const int st = j % CH_STAGES;
    uint8_t* dst = sm + CH_OFF_RING + st * CH_STAGE_BYTES;
    const uint8_t* rec = a.ws + (rec0 + j) * kBlockBytes;
    mbar_arrive_expect_tx(&bars[st], 65536);
    bulk_g2s(dst, rec, 32768, &bars[st]);
    bulk_g2s(dst + 32768, rec + kMBytes + half * 32768, 32768, &bars[st]);
  };
  if (tid == 0)
    for (int j = 0; j < CH_STAGES && j < a.n_blocks; ++j) issue(j);

  // state row a = tid (TMEM lane), columns [64 half, 64 half + 64)
  const int row = tid;
  float S[64];
#pragma unroll
  for (int c = 0; c < 64; ++c)
    S[c] = a.S0 ? a.S0[(((int64_t)b * a.H + h) * D + row) * D + 64 * half + c] : 0.f;

  const uint32_t idesc = idesc_f16(128, 64, false, true);
  auto state_out = [&](int jj) {
    // S (fp16) -> shared B operand and -> workspace (state entering block jj)
    uint8_t* gS = a.ws + (rec0 + jj) * kBlockBytes + kMBytes + kBBytes + kRBytes + kOBytes + half * 16384;
#pragma unroll
    for (int c0 = 0; c0 < 64; c0 += 16) {
      float v[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) v[i] = S[c0 + i];
      st_row16_h(Ssm, row, c0, v);
      st_row16_h(gS, row, c0, v);
    }
    fence_proxy_async();
  };
  state_out(0);
  __syncthreads();
  uint32_t mphase = 0;
  bool ok = true;
  int j = 0;
  for (; j < a.n_blocks; ++j) {
    const int st = j % CH_STAGES;
    uint8_t* stage = sm + CH_OFF_RING + st * CH_STAGE_BYTES;
    bool issued_ok = true;
    if (tid == 0) {
      issued_ok = mbar_wait(&bars[st], (uint32_t)(j / CH_STAGES) & 1u);
      if (issued_ok) {
        fence_after_sync();
        for (int k16 = 0; k16 < 8; ++k16)
          mma_ss(tmem_at(tm, 0, 0), desc_kmajor(smem_u32(stage), k16, 16384), desc_mnmajor(smem_u32(Ssm), k16, 16384),
                 idesc, k16 > 0);
        mma_commit(&bars[3]);
      }
    }
    ok = __syncthreads_and(issued_ok) && ok;
    if (!ok) break;
    const bool done = mbar_wait(&bars[3], mphase);
    mphase ^= 1u;
    ok = __syncthreads_and(done) && ok;
    if (!ok) break;
    fence_after_sync();
    const float4* Bs = reinterpret_cast<const float4*>(stage + 32768);
#pragma unroll
    for (int c0 = 0; c0 < 64; c0 += 32) {
      float v[32];
      tmem_ld32(tmem_at(tm, 32 * warp, c0), v);
      float4 bv[8];
#pragma unroll
      for (int q4 = 0; q4 < 8; ++q4) bv[q4] = Bs[((c0 >> 2) + q4) * 128 + row];
      tmem_wait_ld();
#pragma unroll
      for (int q4 = 0; q4 < 8; ++q4) {
        S[c0 + 4 * q4 + 0] = v[4 * q4 + 0] + bv[q4].x;
        S[c0 + 4 * q4 + 1] = v[4 * q4 + 1] + bv[q4].y;
        S[c0 + 4 * q4 + 2] = v[4 * q4 + 2] + bv[q4].z;
        S[c0 + 4 * q4 + 3] = v[4 * q4 + 3] + bv[q4].w;
      }
    }
    if (j + 1 < a.n_blocks) state_out(j + 1);
    fence_before_sync();
    __syncthreads();   // stage j consumed, TMEM read, next S in shared memory
    if (tid == 0 && j + CH_STAGES < a.n_blocks) issue(j + CH_STAGES);
  }
  if (!ok) {
    if (tid == 0) {
      set_status(a.status, KDA_ERR_TIMEOUT);
      // let copies already issued land before the CTA exits
      const int issued = min(a.n_blocks, j + CH_STAGES);
      for (int jj = j; jj < issued; ++jj) mbar_wait(&bars[jj % CH_STAGES], (uint32_t)(jj / CH_STAGES) & 1u, 100000000ull);
    }
  } else if (a.SN) {
#pragma unroll
    for (int c = 0; c < 64; ++c) a.SN[(((int64_t)b * a.H + h) * D + row) * D + 64 * half + c] = S[c];
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  if (warp == 0) tmem_dealloc(tm, 64);
}

// ---------------------------------------------------------------------------
// kda_tc_out: O = R S + O''
// ---------------------------------------------------------------------------
constexpr uint32_t OUT_SMEM = 65536 + 256 + 1024;

template <typename TOut>
__global__ void __launch_bounds__(128) kda_tc_out(uint8_t* ws, TOut* o, int64_t N, int H, int n_blocks,
                                                  uint32_t* status) {
  extern __shared__ uint8_t dyn[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dyn) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + 65536);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2);
  const int tid = threadIdx.x, warp = tid >> 5;
  const int blk = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const uint8_t* rec = ws + (((int64_t)b * H + h) * n_blocks + blk) * kBlockBytes;
  if (*(volatile uint32_t*)status == KDA_ERR_TIMEOUT) return;   // an earlier CTA gave up: skip the work
  if (warp == 0) { tmem_alloc(tmem_slot, 128); tmem_relinquish(); }
  if (tid == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    fence_mbar_init();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tm = *tmem_slot;
  if (tid == 0) {
    mbar_arrive_expect_tx(&bars[0], 65536);
    bulk_g2s(sm, rec + kMBytes + kBBytes, 32768, &bars[0]);                               // R
    bulk_g2s(sm + 32768, rec + kMBytes + kBBytes + kRBytes + kOBytes, 32768, &bars[0]);   // S
  }
  bool ok = __syncthreads_and(mbar_wait(&bars[0], 0));
  if (ok && tid == 0) {
    fence_after_sync();
    const uint32_t idesc = idesc_f16(128, 128, false, true);
    for (int k16 = 0; k16 < 8; ++k16)
      mma_ss(tm, desc_kmajor(smem_u32(sm), k16, 16384), desc_mnmajor(smem_u32(sm + 32768), k16, 16384), idesc,
             k16 > 0);
    mma_commit(&bars[1]);
  }
  if (ok) ok = __syncthreads_and(mbar_wait(&bars[1], 0));
  if (!ok) {
    if (tid == 0) set_status(status, KDA_ERR_TIMEOUT);
  } else {
    fence_after_sync();
    const int r = tid;  // token row within the block = TMEM lane
    const int64_t tok = (int64_t)blk * BLK + r;
    const float4* Oo = reinterpret_cast<const float4*>(rec + kMBytes + kBBytes + kRBytes);
    TOut* orow = o + ((int64_t)b * N + tok) * H * D + (int64_t)h * D;
    for (int c0 = 0; c0 < 128; c0 += 32) {
      float v[32];
      tmem_ld32(tmem_at(tm, 32 * warp, c0), v);
      float4 oo[8];
#pragma unroll
      for (int q4 = 0; q4 < 8; ++q4) oo[q4] = __ldg(Oo + ((c0 >> 2) + q4) * 128 + r);
      tmem_wait_ld();
      if (tok < N) {
#pragma unroll
        for (int q4 = 0; q4 < 8; ++q4) {
          v[4 * q4] += oo[q4].x; v[4 * q4 + 1] += oo[q4].y; v[4 * q4 + 2] += oo[q4].z; v[4 * q4 + 3] += oo[q4].w;
        }
        uint32_t w[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          __nv_bfloat162 hh = __floats2bfloat162_rn(v[2 * j], v[2 * j + 1]);
          w[j] = *reinterpret_cast<uint32_t*>(&hh);
        }
        uint4* dst = reinterpret_cast<uint4*>(orow + c0);
#pragma unroll
        for (int j = 0; j < 4; ++j) dst[j] = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
      }
    }
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  if (warp == 0) tmem_dealloc(tm, 128);
}

template <typename TIn, typename TOut>
cudaError_t launch_all(const Dims& d, const void* q, const void* k, const void* v, const float* la,
                       const void* beta, const float* S0, void* o, float* SN, uint8_t* ws, uint32_t* status,
                       cudaStream_t s, int* launches) {
  const int n_blocks = (int)((d.N + BLK - 1) / BLK);
  cudaError_t e;
  e = cudaFuncSetAttribute(kda_tc_prep<TIn>, cudaFuncAttributeMaxDynamicSharedMemorySize, PREP_SMEM);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(kda_tc_chain, cudaFuncAttributeMaxDynamicSharedMemorySize, CHAIN_SMEM);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(kda_tc_out<TOut>, cudaFuncAttributeMaxDynamicSharedMemorySize, OUT_SMEM);
  if (e != cudaSuccess) return e;
  PrepArgs pa{q, k, v, la, beta, ws, d.N, d.H, n_blocks, status};
  kda_tc_prep<TIn><<<dim3(n_blocks, d.H, d.B), 256, PREP_SMEM, s>>>(pa);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  ChainArgs ca{ws, S0, SN, d.H, n_blocks, status};
  kda_tc_chain<<<dim3(2, d.H, d.B), 128, CHAIN_SMEM, s>>>(ca);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  kda_tc_out<TOut><<<dim3(n_blocks, d.H, d.B), 128, OUT_SMEM, s>>>(ws, static_cast<TOut*>(o), d.N, d.H, n_blocks,
                                                                   status);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (launches) *launches += 3;
  return cudaSuccess;
}

}  // namespace

size_t chunk_tc_workspace_bytes(const Dims& d) {
  const int64_t n_blocks = (d.N + BLK - 1) / BLK;
  return (size_t)d.B * d.H * n_blocks * kBlockBytes;
}

bool chunk_tc_supported(const Dims& d) { return d.dk == D && d.dv == D; }

cudaError_t launch_chunk_tc(const Dims& d, bool in_f16, const void* q, const void* k, const void* v,
                            const float* log_alpha, const void* beta, const float* S0, void* o, float* SN,
                            void* ws, uint32_t* status, cudaStream_t s, int* launches) {
  // beta and o are bf16 (the problem dtype); q', k', v' are fp16 (internal conv output) or bf16 (caller)
  if (in_f16)
    return launch_all<__half, __nv_bfloat16>(d, q, k, v, log_alpha, beta, S0, o, SN, static_cast<uint8_t*>(ws),
                                             status, s, launches);
  return launch_all<__nv_bfloat16, __nv_bfloat16>(d, q, k, v, log_alpha, beta, S0, o, SN,
                                                  static_cast<uint8_t*>(ws), status, s, launches);
}

}  // namespace kda
