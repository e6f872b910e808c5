// Chunked KDA scan on the sm_100a tensor cores (tcgen05, fp16 operands, fp32
// accumulation in TMEM), for d_k = d_v = 128.
//
// Recurrence (paper.rainbus.top, section 方法步骤详情 step (5)), per head:
//   S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,   o_t = S_t^T q_t.
//
// The sequence is cut into blocks of 128 tokens, each made of two 64-token
// sub-chunks.  Within a sub-chunk, with g_r = sum_{i<=r} log alpha_i (per key
// channel, from the sub-chunk start) and g_l its last value, every factor is a
// product of gates alpha <= 1, so no fp16 operand can overflow, whatever the gates:
//   KG = K e^{g},  QG = Q e^{g},  K~ = K e^{g_l - g},  Gamma = e^{g_l}
//   A  = strict_lower(Diag(beta) [K K^T . e^{g_r - g_i}]),  P = lower([Q K^T . e^{g_r - g_i}])
//   T  = (I + A)^{-1} Diag(beta),  W = T KG,  U~ = T V
//   M_s = Diag(Gamma) - K~^T W,   B_s = K~^T U~,   Q^_s = QG - P W,   O'_s = P U~
// so that, entering with state S, the sub-chunk gives O = Q^_s S + O'_s and
// leaves S <- M_s S + B_s.  The pairwise decays e^{g_r - g_i} of A and P are
// factored at a split point between i and r: a pair (r, i) belongs to the level l
// of the highest bit in which r and i differ, and with s the first token of r's
// half at that level, e^{g_r - g_i} = (prod_{u=s..r} alpha_u)(prod_{u=i+1..s-1} alpha_u).
// Levels 5, 4 and 3 (pairs in different 8-token octets) are three tensor-core
// products; pairs inside an octet are running products on the CUDA cores.
// Two sub-chunks compose into one 128-token block:
//   M = M_2 M_1,  B = M_2 B_1 + B_2,  R = [Q^_1 ; Q^_2 M_1],  O'' = [O'_1 ; Q^_2 B_1 + O'_2]
// and the block maps S to O = R S + O'' and S <- M S + B.
//
// Two kernels:
//   kda_tc_prep   persistent, one CTA per SM, looping over (block, batch item,
//                 head) units: everything above, written to the workspace as one
//                 record per unit (M, B, R, O'' in fp16 operand images).
//   kda_tc_chain  one CTA per (batch item, head, 16, 32 or 64 value columns):
//                 the serial pass S <- M S + B, state kept in registers (fp32),
//                 and beside it the block outputs O = R S + O''.
// Padding tokens of the last block carry k = q = v = 0, beta = 0, log alpha = 0.
#include "common.cuh"
#include "tc.cuh"

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_fp16.h>

#include <mutex>

namespace kda {
namespace {

using namespace tc;

constexpr int BLK = 128;          // tokens per block (one serial step)
constexpr int SUB = 64;           // tokens per sub-chunk
constexpr int D = 128;            // d_k = d_v

// Record per (batch item, head, block), all fp16:
//   M   K-major operand image: 2 panels [128 rows][64 cols]            32 KB
//   B   [c/8][row a][8]  (16-byte units)                               32 KB
//   R   K-major operand image: 2 panels [128 rows][64 cols]            32 KB
//   O'' [row half][c/8][row r % 64][8]  (16-byte units)                32 KB
constexpr size_t kMOff = 0, kBOff = 32768, kROff = 65536, kOOff = 98304;
constexpr size_t kBlockBytes = 131072;

// ---------------------------------------------------------------------------
// small helpers
// ---------------------------------------------------------------------------
template <typename T> constexpr bool kIsHalf = false;
template <> constexpr bool kIsHalf<__half> = true;

__device__ __forceinline__ void st_h2(uint8_t* p, float a, float b) {
  *reinterpret_cast<__half2*>(p) = __floats2half2_rn(a, b);
}
__device__ __forceinline__ uint32_t pack_h2(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ uint4 pack8(const float* v) {
  return make_uint4(pack_h2(v[0], v[1]), pack_h2(v[2], v[3]), pack_h2(v[4], v[5]), pack_h2(v[6], v[7]));
}
__device__ __forceinline__ void unpack8(uint4 u, float* v) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}

// 32 consecutive fp32 values -> fp16 at (row, col0..col0+31) of a swizzled
// panel (col0 a multiple of 32).  Eight consecutive rows writing the same chunk
// land in eight different bank groups (the swizzle), so stores need no reordering.
__device__ __forceinline__ void st_row32_h(uint8_t* panel, int row, int col0, const float (&v)[32]) {
#pragma unroll
  for (int c = 0; c < 4; ++c) *reinterpret_cast<uint4*>(panel + swz_off(row, col0 + 8 * c)) = pack8(v + 8 * c);
}
// 16 consecutive fp16 values at (row, col0..) of a swizzled panel -> fp32
__device__ __forceinline__ void ld_row16_h(const uint8_t* panel, int row, int col0, float* v) {
  unpack8(*reinterpret_cast<const uint4*>(panel + swz_off(row, col0)), v);
  unpack8(*reinterpret_cast<const uint4*>(panel + swz_off(row, col0 + 8)), v + 8);
}

// 16 or 32 consecutive TMEM columns of this warp's lanes
template <int N>
__device__ __forceinline__ void tmem_ld_n(uint32_t taddr, float (&v)[N]) {
  static_assert(N == 16 || N == 32, "16 or 32 columns");
  if constexpr (N == 16) tmem_ld16(taddr, v); else tmem_ld32(taddr, v);
}

__device__ __forceinline__ uint32_t tmem_at(uint32_t base, int lane0, int col) {
  return base + ((uint32_t)lane0 << 16) + (uint32_t)col;
}

// Waits (at most tmo ns) for a TMA load counted on `bar`; on timeout records the status.
// Returns false on timeout.
__device__ __forceinline__ bool wait_tma(uint64_t* bar, uint32_t& phase, uint32_t* status, bool alive, uint64_t tmo) {
  if (!alive) return false;
  const bool ok = mbar_wait(bar, phase, tmo);
  if (ok) phase ^= 1u;
  else set_status(status, KDA_ERR_TIMEOUT);
  return ok;
}

// Waits (at most tmo ns) on the MMA barrier; on timeout records the status.  Returns false on timeout.
__device__ __forceinline__ bool wait_mma(uint64_t* bar, uint32_t& phase, uint32_t* status, bool alive, uint64_t tmo) {
  if (!alive) return false;   // nothing was issued
  const bool ok = mbar_wait(bar, phase, tmo);
  phase ^= 1u;
  if (!ok) set_status(status, KDA_ERR_TIMEOUT);
  return ok;
}

// ---------------------------------------------------------------------------
// kda_tc_prep
// ---------------------------------------------------------------------------
// shared memory map (bytes from a 1024-aligned base)
constexpr uint32_t OFF_KQ = 0;          // [128 rows][128] fp16: rows 0-63 K -> K Gamma (later W), 64-127 Q -> Q Gamma; later M_2
constexpr uint32_t OFF_KN = 32768;      // [64][128] fp16: K~; staging of O'_1 and O''_2
constexpr uint32_t OFF_VV = 49152;      // [64][128] fp16: V, then U~, then Q^_2
constexpr uint32_t OFF_TT = 65536;      // [64][64] fp16: T   (TT and PP together: staging of R_1 and R_2)
constexpr uint32_t OFF_PP = 73728;      // [64][64] fp16: P
constexpr uint32_t OFF_M1 = 81920;      // [128][128] fp16: M_1 (MN-major operand image)
constexpr uint32_t OFF_B1 = 114688;     // [128][128] fp16: B_1 (MN-major operand image)
// 72 KB used three ways in turn: the log alpha of a sub-chunk (TMA target, [64 tokens][128] fp32), the
// operand tiles of the three tensor-core Gram levels, and A, X, Y of the blocked inverse
constexpr uint32_t OFF_G = 147456;
constexpr uint32_t G_ROW = 0;           // level tiles, rows: [64][128] fp16 per level (5, 4, 3), 16 KB apart
constexpr uint32_t G_COL = 49152;       // level tiles, columns: [32][128] fp16 per level, 8 KB apart
constexpr uint32_t G_AS = 0;            // fp32 [64][LDA]: A (strictly lower, beta applied)
constexpr uint32_t G_XS = 17408;        // fp32 [64][LDXS]: (I + A)^{-1}
constexpr uint32_t G_YS = 34816;        // fp32 [32][36]: merge scratch
constexpr uint32_t OFF_MISC = OFF_G + 73728;   // beta[64], Gamma_l[128], octet totals [8][128], octet Gram [8][64], barriers
constexpr uint32_t PREP_SMEM = OFF_MISC + 8192 + 1024;   // + alignment slack

constexpr int LDA = 68;    // row stride of A: rows 16-byte aligned (4-wide stores and loads)
constexpr int LDXS = 68;   // row stride of X: rows 16-byte aligned for 4-wide loads
static_assert(G_XS >= G_AS + 64 * LDA * 4 && G_YS >= G_XS + 64 * LDXS * 4 && G_YS + 32 * 36 * 4 <= 73728,
              "prep shared-memory map");
static_assert(G_COL >= G_ROW + 3 * 16384 && G_COL + 3 * 8192 <= 73728, "prep shared-memory map");
static_assert(PREP_SMEM <= 232448, "prep shared memory above the per-block limit");
constexpr int LDY = 36;    // row stride of the merge scratch

// TMEM columns
constexpr int C_G = 0;                   // the three Gram levels, 32 columns each (M = 64 layout)
constexpr int C_W = 64, C_U = 192;
constexpr int C_MK = 0, C_BK = 128, C_PW = 256, C_PU = 384;

// TMA descriptors of the [B][N][H][128] inputs, box [1][64 tokens][1][64 or 128 channels]
struct PrepMaps {
  CUtensorMap q, k, v;   // 64-channel boxes, 128-byte swizzle: one operand panel each
  CUtensorMap la;        // 128-channel box, no swizzle
};

struct PrepArgs {
  const void* q; const void* k; const void* v;
  const float* la; const void* beta;
  uint8_t* ws;            // block records
  int64_t N; int H; int BH; int n_blocks; int n_units;
  uint32_t* status;
  uint64_t wait_ns;       // limit of every device wait
  int fault;              // self-test: 1 = the first CTA never issues its first k/q/v load
};

// One 16x8 tile of C = A B with fp32 operands in shared memory (A row-major with
// leading dimension lda, 16 rows; B row-major [k][n] with leading dimension ldb,
// 8 columns), K = 8 * ksteps, on mma.sync m16n8k8 tf32 with the operands split
// as x = hi + lo (both tf32): C = A_hi B_hi + A_hi B_lo + A_lo B_hi.  Fragment
// coordinates: g = lane / 4, t = lane % 4; d[0..3] = C[g][2t], C[g][2t+1],
// C[g+8][2t], C[g+8][2t+1].
// x with its 13 low mantissa bits cleared: a tf32 value; applied to x and to the exact
// remainder x - hi it splits x into two tf32 terms (dropped bits below 2^-20 of |x|)
__device__ __forceinline__ uint32_t tf32_hi(float x) { return __float_as_uint(x) & 0xffffe000u; }
__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
  asm volatile("mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
               : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
               : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}
__device__ __forceinline__ void mma_tile_3xtf32(const float* A, int lda, const float* B, int ldb, int ksteps, int g,
                                                int t, float (&d)[4]) {
  // four independent accumulation chains (even / odd k-steps, main / correction terms),
  // summed at the end, so consecutive products do not wait on each other
  float dh[2][4] = {}, dl[2][4] = {};
#pragma unroll
  for (int kk = 0; kk < ksteps; ++kk) {
    const float af[4] = {A[g * lda + 8 * kk + t], A[(g + 8) * lda + 8 * kk + t], A[g * lda + 8 * kk + t + 4],
                         A[(g + 8) * lda + 8 * kk + t + 4]};
    const float bf[2] = {B[(8 * kk + t) * ldb + g], B[(8 * kk + t + 4) * ldb + g]};
    uint32_t ah[4], al[4], bh[2], bl[2];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      ah[i] = tf32_hi(af[i]);
      al[i] = tf32_hi(af[i] - __uint_as_float(ah[i]));
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      bh[i] = tf32_hi(bf[i]);
      bl[i] = tf32_hi(bf[i] - __uint_as_float(bh[i]));
    }
    mma_tf32(dl[kk & 1], al, bh);
    mma_tf32(dl[kk & 1], ah, bl);
    mma_tf32(dh[kk & 1], ah, bh);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) d[i] = (dl[0][i] + dl[1][i]) + (dh[0][i] + dh[1][i]);
}

// Blocked inverse X = (I + A)^{-1} of the unit lower-triangular 64x64 matrix,
// A strictly lower in As, delivered as T = X Diag(beta) in fp16 (TT, one
// swizzled K-major panel).  16x16 diagonal blocks by forward substitution, then
// two doubling merges (X_21 = -X_22 A_21 X_11) at 32 and 64.  Every loop has a
// fixed trip count; the zero blocks above the diagonal of X_11 and X_22 are
// written here, the rest of the upper triangle is never read.
// Step 1 (inverse_diag32) leaves the two diagonal 32x32 blocks of X in Xs and
// writes every part of T but its lower-left block, so products over T's
// columns 32-63 can start while step 2 (inverse_merge64) forms that block.
__device__ void inverse_diag32(const float* As, float* Xs, float* Ys, uint8_t* TT, const float* beta) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (warp < 4 && lane < 16) {
    // diagonal block `warp`, column `lane`: right-looking substitution
    const int o = 16 * warp, l = lane;
    float x[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) x[r] = r == l ? 1.f : 0.f;
    // row r: x[r] -= A[r][m] x[m] for m = 0 .. r-1 in that order, A's row read 4 wide
#pragma unroll
    for (int r = 1; r < 16; ++r) {
      const float4* arow = reinterpret_cast<const float4*>(As + (o + r) * LDA + o);
#pragma unroll
      for (int q = 0; q < (r + 3) / 4; ++q) {
        const float4 a4 = arow[q];
        const float av[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (4 * q + u < r) x[r] -= av[u] * x[4 * q + u];
      }
    }
#pragma unroll
    for (int r = 0; r < 16; ++r) Xs[(o + r) * LDXS + o + l] = x[r];
  } else if (warp >= 4) {
    // zero blocks (0,1) and (2,3)
    const int e = tid - 128, r = e >> 3, c = 2 * (e & 7);   // 16 rows x 8 column pairs
    Xs[r * LDXS + 16 + c] = 0.f;
    Xs[r * LDXS + 17 + c] = 0.f;
    Xs[(32 + r) * LDXS + 48 + c] = 0.f;
    Xs[(32 + r) * LDXS + 49 + c] = 0.f;
  }
  __syncthreads();
  {
    // 32-merges p = 0, 1: X[32p+16.., 32p..] = -D_{2p+1} (A_{2p+1,2p} D_{2p}); 2x1 outputs per thread
    const int p = tid >> 7, e = tid & 127;
    const int o = 32 * p, i0 = 2 * (e >> 4), j = e & 15;
    float* Y = Ys + p * 16 * 17;
    float y0 = 0.f, y1 = 0.f;
#pragma unroll
    for (int m = 0; m < 16; ++m) {
      const float d = Xs[(o + m) * LDXS + o + j];
      y0 += As[(o + 16 + i0) * LDA + o + m] * d;
      y1 += As[(o + 17 + i0) * LDA + o + m] * d;
    }
    Y[i0 * 17 + j] = y0;
    Y[(i0 + 1) * 17 + j] = y1;
    __syncthreads();
    float z0 = 0.f, z1 = 0.f;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const float y = Y[k * 17 + j];
      z0 += Xs[(o + 16 + i0) * LDXS + o + 16 + k] * y;
      z1 += Xs[(o + 17 + i0) * LDXS + o + 16 + k] * y;
    }
    Xs[(o + 16 + i0) * LDXS + o + j] = -z0;
    Xs[(o + 17 + i0) * LDXS + o + j] = -z1;
  }
  __syncthreads();
  // T = X Diag(beta) for rows 0-31 (X_11, then zeros) and the X_22 block of rows 32-63
  for (int e = tid; e < 384; e += 256) {
    const int r = e < 256 ? e >> 3 : 32 + ((e - 256) >> 2);
    const int c0 = e < 256 ? (e & 7) * 8 : 32 + ((e - 256) & 3) * 8;
    float v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int cj = c0 + j;
      v[j] = (cj <= r && (r < 32) == (cj < 32)) ? Xs[r * LDXS + cj] * beta[cj] : 0.f;
    }
    *reinterpret_cast<uint4*>(TT + swz_off(r, c0)) = pack8(v);
  }
  fence_proxy_async();
}

// Step 2: X_21 = -X_22 (A_21 X_11) -> T rows 32-63, columns 0-31.  `between`
// runs on every thread after the barrier that follows the first product; the
// caller's next barrier publishes the block.
template <typename F>
__device__ __forceinline__ void inverse_merge64(const float* As, const float* Xs, float* Ys, uint8_t* TT,
                                                const float* beta, F&& between) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  {
    // 64-merge: X[32.., 0..31] = -X_22 (A_21 X_11), two 32x32x32 products on the
    // warp-level tensor cores (m16n8k8, tf32).  Each operand is split into a tf32
    // high part and a tf32 remainder and the product is formed as hi*hi + hi*lo +
    // lo*hi, which keeps it at about fp32 accuracy.  Warp w owns the 16x8 output
    // tile (rows 16*(w>>2), columns 8*(w&3)).
    const int g = lane >> 2, t4 = lane & 3;
    const int tm = warp >> 2, tn = warp & 3;
    float d[4];
    // Y = A_21 X_11 -> Ys
    mma_tile_3xtf32(As + (32 + 16 * tm) * LDA, LDA, Xs + 8 * tn, LDXS, 4, g, t4, d);
    Ys[(16 * tm + g) * LDY + 8 * tn + 2 * t4] = d[0];
    Ys[(16 * tm + g) * LDY + 8 * tn + 2 * t4 + 1] = d[1];
    Ys[(16 * tm + g + 8) * LDY + 8 * tn + 2 * t4] = d[2];
    Ys[(16 * tm + g + 8) * LDY + 8 * tn + 2 * t4 + 1] = d[3];
    __syncthreads();
    between();
    // X_21 = -X_22 Y, times beta of its column, into T
    mma_tile_3xtf32(Xs + (32 + 16 * tm) * LDXS + 32, LDXS, Ys + 8 * tn, LDY, 4, g, t4, d);
    const int r0 = 32 + 16 * tm + g, c = 8 * tn + 2 * t4;
    const float b0 = beta[c], b1 = beta[c + 1];
    st_h2(TT + swz_off(r0, c), -d[0] * b0, -d[1] * b1);
    st_h2(TT + swz_off(r0 + 8, c), -d[2] * b0, -d[3] * b1);
    fence_proxy_async();
  }
}

// 4 consecutive activations (8 bytes, fp16 or bf16) -> fp32, and 4 fp32 -> fp16 (8 bytes)
__device__ __forceinline__ void ld_act4(const uint8_t* p, float* v, __half*) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&u.x));
  const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&u.y));
  v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
}
__device__ __forceinline__ void ld_act4(const uint8_t* p, float* v, __nv_bfloat16*) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
  v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
}
__device__ __forceinline__ void st_h4(uint8_t* p, float a, float b, float c, float d) {
  *reinterpret_cast<uint2*>(p) = make_uint2(pack_h2(a, b), pack_h2(c, d));
}

// Position of token t (0..63) among the 32 tokens of its role at Gram level l: the
// tokens whose bit l is set (rows) or clear (columns), in increasing order.
__device__ __forceinline__ int level_pos(int t, int l) { return ((t >> (l + 1)) << l) | (t & ((1 << l) - 1)); }

// v[0..N-1] summed over the 32 lanes of a warp, scattered: lane L ends with the
// totals of v[2L] and v[2L + 1] (for N = 64) in v[0] and v[1].  Each round keeps the
// half of the vector that the lane's bit S selects and adds the partner's copy of it.
template <int S, int N>
__device__ __forceinline__ void reduce_scatter_round(float (&v)[64], int lane) {
  const bool up = (lane & S) != 0;
#pragma unroll
  for (int x = 0; x < N / 2; ++x) {
    const float lo = v[x], hi = v[x + N / 2];
    const float keep = up ? hi : lo, send = up ? lo : hi;
    v[x] = keep + __shfl_xor_sync(0xffffffffu, send, S);
  }
}
__device__ __forceinline__ void warp_reduce_scatter64(float (&v)[64], int lane) {
  reduce_scatter_round<16, 64>(v, lane);
  reduce_scatter_round<8, 32>(v, lane);
  reduce_scatter_round<4, 16>(v, lane);
  reduce_scatter_round<2, 8>(v, lane);
  reduce_scatter_round<1, 4>(v, lane);
}

// Index of a pair (r, i) of one octet in the octet Gram: A pairs i < r at r(r-1)/2 + i
// (28 of them), P pairs i <= r at 28 + r(r+1)/2 + i (36).
__host__ __device__ constexpr int oct_a(int r, int i) { return r * (r - 1) / 2 + i; }
__host__ __device__ constexpr int oct_p(int r, int i) { return 28 + r * (r + 1) / 2 + i; }

template <typename TIn>
__global__ void __launch_bounds__(256, 1) kda_tc_prep(PrepArgs a, const __grid_constant__ PrepMaps mp) {
  extern __shared__ uint8_t dyn[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dyn) + 1023) & ~uintptr_t(1023));
  uint8_t* KQ = sm + OFF_KQ;
  uint8_t* KN = sm + OFF_KN;
  uint8_t* VV = sm + OFF_VV;
  uint8_t* TT = sm + OFF_TT;
  uint8_t* PP = sm + OFF_PP;
  uint8_t* M1 = sm + OFF_M1;
  uint8_t* B1 = sm + OFF_B1;
  uint8_t* G = sm + OFF_G;
  const float* LA = reinterpret_cast<const float*>(G);      // log alpha of the sub-chunk (TMA)
  float* As = reinterpret_cast<float*>(G + G_AS);
  float* Xs = reinterpret_cast<float*>(G + G_XS);
  float* Ys = reinterpret_cast<float*>(G + G_YS);
  float* beta_s = reinterpret_cast<float*>(sm + OFF_MISC);  // 64
  float* egl = beta_s + 64;                                 // 128: Gamma_l = e^{g_l}
  float* tot = egl + 128;                                   // [8 octets][128]: decay over each octet
  float* gscr = tot + 8 * 128;                              // [8 octets][64]: Gram pairs inside each octet
  uint64_t* bar = reinterpret_cast<uint64_t*>(gscr + 8 * 64);   // [0] MMA, [1] k/q/v tiles, [2] log alpha
  uint64_t* kqv_bar = bar + 1;
  uint64_t* la_bar = bar + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int sub = warp & 3, chalf = warp >> 2;

  if (*(volatile uint32_t*)a.status == KDA_ERR_TIMEOUT) return;   // an earlier CTA gave up: skip the work
  if (warp == 0) { tmem_alloc(tmem_slot, 512); tmem_relinquish(); }
  if (tid == 0) {
    mbar_init(bar, 1);
    mbar_init(kqv_bar, 1);
    mbar_init(la_bar, 1);
    fence_mbar_init();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tm = *tmem_slot;
  uint32_t phase = 0, kqv_phase = 0, la_phase = 0;
  bool alive = true;
  bool la_inflight = false, kqv_inflight = false;   // thread 0's view: TMA loads not yet waited for
  // batch item, head and first token of the sub-chunk this CTA processes after (u, s_)
  auto next_sub = [&](int u, int s_, int& nb_, int& nh_, int& nt0_) -> bool {
    const int nu = s_ == 0 ? u : u + (int)gridDim.x;
    if (nu >= a.n_units) return false;
    const int blk_ = nu / a.BH, bh_ = nu - blk_ * a.BH;
    nb_ = bh_ / a.H;
    nh_ = bh_ - nb_ * a.H;
    nt0_ = blk_ * BLK + (s_ ^ 1) * SUB;
    return true;
  };
  auto load_beta = [&](int b_, int h_, int t_) -> float {   // 0 past the sequence end
    return t_ < a.N ? __bfloat162float(static_cast<const __nv_bfloat16*>(a.beta)[((int64_t)b_ * a.N + t_) * a.H + h_])
                    : 0.f;
  };
  float beta_next = 0.f;
  if (tid < SUB && (int)blockIdx.x < a.n_units) {
    const int bh_ = (int)blockIdx.x % a.BH;   // unit blockIdx.x: block blockIdx.x / BH, sub-chunk 0
    beta_next = load_beta(bh_ / a.H, bh_ % a.H, ((int)blockIdx.x / a.BH) * BLK + tid);
  }
  // k, q, v of the sub-chunk starting at token t0_ -> KQ rows 0-63 / 64-127 and VV (thread 0)
  auto issue_kqv = [&](int b_, int h_, int t0_) {
    mbar_arrive_expect_tx(kqv_bar, 6 * 8192);
#pragma unroll
    for (int pnl = 0; pnl < 2; ++pnl) {
      tma_load_4d(KQ + pnl * 16384, &mp.k, 64 * pnl, h_, t0_, b_, kqv_bar);
      tma_load_4d(KQ + pnl * 16384 + 8192, &mp.q, 64 * pnl, h_, t0_, b_, kqv_bar);
      tma_load_4d(VV + pnl * 8192, &mp.v, 64 * pnl, h_, t0_, b_, kqv_bar);
    }
  };
  bool kqv_early = false;   // thread 0: the next sub-chunk's tiles are already on their way
  auto issue_la = [&](int u, int s_) {   // log alpha of sub-chunk s_ of unit u -> G (thread 0)
    const int blk_ = u / a.BH, bh_ = u - blk_ * a.BH;
    const int b_ = bh_ / a.H, h_ = bh_ - b_ * a.H;
    mbar_arrive_expect_tx(la_bar, 32768);
    tma_load_4d(G, &mp.la, 0, h_, blk_ * BLK + s_ * SUB, b_, la_bar);
  };
  if (tid == 0 && (int)blockIdx.x < a.n_units) {
    issue_la(blockIdx.x, 0);
    la_inflight = true;
  }

  // operand descriptors of the fixed tiles (stepped along K by kstep / mstep)
  const uint64_t dKQk = kdesc0(smem_u32(KQ)), dKQm = mdesc0(smem_u32(KQ), 16384);
  const uint64_t dKNm = mdesc0(smem_u32(KN), 8192);
  const uint64_t dVVk = kdesc0(smem_u32(VV)), dVVm = mdesc0(smem_u32(VV), 8192);
  const uint64_t dTTk = kdesc0(smem_u32(TT)), dPPk = kdesc0(smem_u32(PP));
  const uint64_t dM1m = mdesc0(smem_u32(M1), 16384), dB1m = mdesc0(smem_u32(B1), 16384);
  const uint64_t dGrow = kdesc0(smem_u32(G + G_ROW)), dGcol = kdesc0(smem_u32(G + G_COL));
  const uint32_t id_gram = idesc_f16(64, 32, false, false);
  const uint32_t id_64x128_kmn = idesc_f16(64, 128, false, true);
  const uint32_t id_128x128_mnmn = idesc_f16(128, 128, true, true);
  const uint32_t id_128x128_kmn = idesc_f16(128, 128, false, true);

  // front-pass role of this thread: octet fo (tokens 8 fo .. 8 fo + 7), channels 4 lane .. 4 lane + 3
  const int fo = warp, fpnl = lane >> 4, fpc = (4 * lane) & 63;

  for (int unit = blockIdx.x; unit < a.n_units && alive; unit += gridDim.x) {
    const int blk = unit / a.BH, bh = unit - blk * a.BH;
    const int b = bh / a.H, h = bh - b * a.H;
    uint8_t* rec = a.ws + (((int64_t)b * a.H + h) * a.n_blocks + blk) * kBlockBytes;
    uint8_t* gM = rec + kMOff;
    uint8_t* gB = rec + kBOff;
    uint8_t* gR = rec + kROff;
    uint8_t* gO = rec + kOOff;

    for (int s = 0; s < 2; ++s) {
      const int64_t t0 = (int64_t)blk * BLK + s * SUB;
      // ---------------- inputs ----------------
      // k -> KQ rows 0-63, q -> KQ rows 64-127, v -> VV: 128-byte-swizzled operand panels
      // written by TMA; rows past the sequence end read as zero (log alpha too: alpha = 1)
      if (tid == 0 && alive) {
        // self-test of the bounded waits: a load that is never issued, so the wait below gives up
        const bool skip = a.fault == 1 && blockIdx.x == 0 && unit == 0 && s == 0;
        if (!kqv_early && !skip) issue_kqv(b, h, (int)t0);   // else issued while the previous unit finished
        kqv_early = false;
        kqv_inflight = !skip;
      }
      if (tid == 128 && alive) {
        // the next sub-chunk's tiles and log alpha into L2 meanwhile
        int nb_, nh_, nt0_;
        if (next_sub(unit, s, nb_, nh_, nt0_)) {
#pragma unroll
          for (int pnl = 0; pnl < 2; ++pnl) {
            tma_prefetch_4d(&mp.k, 64 * pnl, nh_, nt0_, nb_);
            tma_prefetch_4d(&mp.q, 64 * pnl, nh_, nt0_, nb_);
            tma_prefetch_4d(&mp.v, 64 * pnl, nh_, nt0_, nb_);
          }
          tma_prefetch_4d(&mp.la, 0, nh_, nt0_, nb_);
        }
      }
      if (tid < SUB) {
        // beta of this sub-chunk was read one sub-chunk ago; read the next one now
        beta_s[tid] = beta_next;
        int nb_, nh_, nt0_;
        beta_next = next_sub(unit, s, nb_, nh_, nt0_) ? load_beta(nb_, nh_, nt0_ + tid) : 0.f;
      }
      {
        const bool ok_la = wait_tma(la_bar, la_phase, a.status, alive, a.wait_ns);
        const bool ok_kqv = wait_tma(kqv_bar, kqv_phase, a.status, ok_la, a.wait_ns);
        if (tid == 0) {
          if (ok_la) la_inflight = false;
          if (ok_kqv) kqv_inflight = false;
        }
        alive = __syncthreads_and(ok_kqv);
      }
      // ---------------- front pass ----------------
      // Every factor is a product of gates alpha = e^{log alpha} <= 1, so none can overflow:
      //   Gamma_t = prod_{u<=t} alpha_u,  e^{g_l - g_t} = prod_{u>t} alpha_u,
      // and the Gram levels' factors, prefix products from a split point (rows) and suffix
      // products up to it (columns).  Thread: octet fo, four channels; within the octet the
      // prefix (pre) and suffix (suf) products are its own, across octets it uses the octet totals.
      float al[8][4], kx[8][4], qx[8][4];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int tok = 8 * fo + j;
        const float4 x = *reinterpret_cast<const float4*>(LA + tok * D + 4 * lane);
        al[j][0] = __expf(x.x); al[j][1] = __expf(x.y); al[j][2] = __expf(x.z); al[j][3] = __expf(x.w);
        ld_act4(KQ + fpnl * 16384 + swz_off(tok, fpc), kx[j], (TIn*)nullptr);
        ld_act4(KQ + fpnl * 16384 + swz_off(64 + tok, fpc), qx[j], (TIn*)nullptr);
        if constexpr (!kIsHalf<TIn>) {   // caller's bf16 v -> the fp16 operand image, in place
          uint8_t* pv = VV + fpnl * 8192 + swz_off(tok, fpc);
          float v4[4];
          ld_act4(pv, v4, (TIn*)nullptr);
          st_h4(pv, v4[0], v4[1], v4[2], v4[3]);
        }
      }
      float pre[8][4], suf[8][4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        pre[0][c] = al[0][c];
#pragma unroll
        for (int j = 1; j < 8; ++j) pre[j][c] = pre[j - 1][c] * al[j][c];
        suf[7][c] = 1.f;
#pragma unroll
        for (int j = 6; j >= 0; --j) suf[j][c] = suf[j + 1][c] * al[j + 1][c];
      }
      *reinterpret_cast<float4*>(tot + fo * D + 4 * lane) = make_float4(pre[7][0], pre[7][1], pre[7][2], pre[7][3]);
      if (tid == 0) bulk_wait_read();   // staged record stores have read KN, TT and PP
      __syncthreads();                  // octet totals published; log alpha read (G is free)
      {
        // outer factors from the octet totals (fo is uniform over the warp)
        float gb[4], ka[4], f5[4], f4[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) gb[c] = ka[c] = f5[c] = f4[c] = 1.f;
#pragma unroll
        for (int o = 0; o < 8; ++o) {
          const float4 t4 = *reinterpret_cast<const float4*>(tot + o * D + 4 * lane);
          const float tv[4] = {t4.x, t4.y, t4.z, t4.w};
          const bool in5 = (fo & 4) ? (o >= 4 && o < fo) : (o > fo && o < 4);
          const bool in4 = (fo & 2) ? ((fo & 1) && o == fo - 1) : (!(fo & 1) && o == fo + 1);
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            if (o < fo) gb[c] *= tv[c];
            if (o > fo) ka[c] *= tv[c];
            if (in5) f5[c] *= tv[c];
            if (in4) f4[c] *= tv[c];
          }
          if (fo == 0) {
            // Gamma_l: the decay over the whole sub-chunk
            if (o == 0) *reinterpret_cast<float4*>(egl + 4 * lane) = t4;
            else {
              float4 e = *reinterpret_cast<const float4*>(egl + 4 * lane);
              e.x *= t4.x; e.y *= t4.y; e.z *= t4.z; e.w *= t4.w;
              *reinterpret_cast<float4*>(egl + 4 * lane) = e;
            }
          }
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int tok = 8 * fo + j;
          float g[4], kt[4], r3[4], r4[4], r5[4];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            g[c] = gb[c] * pre[j][c];
            kt[c] = suf[j][c] * ka[c];
            r3[c] = (fo & 1) ? pre[j][c] : suf[j][c];
            r4[c] = (fo & 2) ? f4[c] * pre[j][c] : suf[j][c] * f4[c];
            r5[c] = (fo & 4) ? f5[c] * pre[j][c] : suf[j][c] * f5[c];
          }
          const float* kk = kx[j];
          const float* qq = qx[j];
          const uint32_t o128 = swz_off(tok, fpc);
          st_h4(KQ + fpnl * 16384 + o128, kk[0] * g[0], kk[1] * g[1], kk[2] * g[2], kk[3] * g[3]);
          st_h4(KQ + fpnl * 16384 + swz_off(64 + tok, fpc), qq[0] * g[0], qq[1] * g[1], qq[2] * g[2], qq[3] * g[3]);
          st_h4(KN + fpnl * 8192 + o128, kk[0] * kt[0], kk[1] * kt[1], kk[2] * kt[2], kk[3] * kt[3]);
          // Gram levels 5, 4, 3 (tile li = 5 - level): role from bit `level` of the token
#pragma unroll
          for (int li = 0; li < 3; ++li) {
            const int lvl = 5 - li;
            const float* f = li == 0 ? r5 : (li == 1 ? r4 : r3);
            const int pos = level_pos(tok, lvl);
            if ((tok >> lvl) & 1) {
              uint8_t* rt = G + G_ROW + li * 16384 + fpnl * 8192;
              st_h4(rt + swz_off(pos, fpc), kk[0] * f[0], kk[1] * f[1], kk[2] * f[2], kk[3] * f[3]);
              st_h4(rt + swz_off(32 + pos, fpc), qq[0] * f[0], qq[1] * f[1], qq[2] * f[2], qq[3] * f[3]);
            } else {
              uint8_t* ct = G + G_COL + li * 8192 + fpnl * 4096;
              st_h4(ct + swz_off(pos, fpc), kk[0] * f[0], kk[1] * f[1], kk[2] * f[2], kk[3] * f[3]);
            }
          }
        }
      }
      fence_proxy_async();
      fence_before_sync();
      __syncthreads();
      // ---------------- Gram levels on the tensor cores ----------------
      // Level l pairs the 32 tokens with bit l set (rows: k and q, scaled by the decay from
      // the level's split point) with the 32 with bit l clear (columns: k, scaled by the
      // decay up to it): entry (r, i) is valid when r and i share their bits above l, and
      // then equals sum_c k_r (or q_r) k_i e^{g_r - g_i}.  Levels 5, 4, 3 cover every pair
      // in different octets; pairs inside an octet follow on the CUDA cores.
      if (tid == 0 && alive) {
        fence_after_sync();
#pragma unroll
        for (int li = 0; li < 3; ++li)
#pragma unroll
          for (int k16 = 0; k16 < 8; ++k16)
            mma_ss(tmem_at(tm, 0, C_G + 32 * li), dGrow + ((uint32_t)li * 16384 >> 4) + kstep(k16, 8192),
                   dGcol + ((uint32_t)li * 8192 >> 4) + kstep(k16, 4096), id_gram, k16 > 0);
        mma_commit(bar);
      }
      {
        // pairs inside the octet: e^{g_r - g_i} = prod_{u=i+1..r} alpha_u as a running product
        float acc[64];
#pragma unroll
        for (int x = 0; x < 64; ++x) acc[x] = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            float kf = kx[i][c];
            acc[oct_p(i, i)] += qx[i][c] * kf;
#pragma unroll
            for (int r = i + 1; r < 8; ++r) {
              kf *= al[r][c];
              acc[oct_a(r, i)] += kx[r][c] * kf;
              acc[oct_p(r, i)] += qx[r][c] * kf;
            }
          }
        }
        warp_reduce_scatter64(acc, lane);
        *reinterpret_cast<float2*>(gscr + fo * 64 + 2 * lane) = make_float2(acc[0], acc[1]);
      }
      alive = __syncthreads_and(wait_mma(bar, phase, a.status, alive, a.wait_ns));
      fence_after_sync();
      {
        // Gram levels -> A (fp32, beta applied, As) and P (fp16, PP).  M = 64 accumulator layout:
        // row m at lane 32 (m / 16) + m % 16; rows 0-31 are k rows (A), 32-63 q rows (P).
        const int qd = warp & 3;
        const bool isP = qd >= 2;
        const int mr = 16 * (qd & 1) + lane;   // row among the 32 of its kind (lanes < 16)
        auto put = [&](int r, int i0, const float* v, int n) {   // n = 8, 16 or 32 consecutive columns
          if (!isP) {
            const float bt = beta_s[r];
#pragma unroll
            for (int j = 0; j < n; j += 4)
              *reinterpret_cast<float4*>(As + r * LDA + i0 + j) =
                  make_float4(bt * v[j], bt * v[j + 1], bt * v[j + 2], bt * v[j + 3]);
          } else {
#pragma unroll
            for (int j = 0; j < n; j += 8) *reinterpret_cast<uint4*>(PP + swz_off(r, i0 + j)) = pack8(v + j);
          }
        };
        if (warp < 4) {
          float v[32];   // level 5: rows 32..63 against columns 0..31, all valid
          tmem_ld32(tmem_at(tm, 32 * qd, C_G), v);
          tmem_wait_ld();
          if (lane < 16) put(32 + mr, 0, v, 32);
        } else {
          float v4[16], v3[16];
          // level 4: this warp's 16 rows share one 16-column block; level 3: two 8-column blocks
          tmem_ld16(tmem_at(tm, 32 * qd, C_G + 32 + 16 * (qd & 1)), v4);
          tmem_ld16(tmem_at(tm, 32 * qd, C_G + 64 + 16 * (qd & 1)), v3);
          tmem_wait_ld();
          if (lane < 16) {
            put(((mr >> 4) << 5) | 16 | (mr & 15), 32 * (mr >> 4), v4, 16);
            float w8[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) w8[c] = (lane & 8) ? v3[8 + c] : v3[c];
            put(((mr >> 3) << 4) | 8 | (mr & 7), 16 * (mr >> 3), w8, 8);
          }
        }
        if (tid < SUB) {
          // row r: the pairs inside its octet, and zeros above the diagonal of P
          const int r = tid, o = r >> 3, jr = r & 7;
          const float bt = beta_s[r];
          const float* gs = gscr + o * 64;
          for (int ji = 0; ji < jr; ++ji) As[r * LDA + 8 * o + ji] = bt * gs[oct_a(jr, ji)];
          float pv[8];
#pragma unroll
          for (int ji = 0; ji < 8; ++ji) pv[ji] = ji <= jr ? gs[oct_p(jr, ji)] : 0.f;
          *reinterpret_cast<uint4*>(PP + swz_off(r, 8 * o)) = pack8(pv);
          for (int c8 = o + 1; c8 < 8; ++c8) *reinterpret_cast<uint4*>(PP + swz_off(r, 8 * c8)) = make_uint4(0, 0, 0, 0);
        }
      }
      fence_proxy_async();
      fence_before_sync();
      __syncthreads();
      // T = (I + A)^{-1} Diag(beta) -> TT; W = T K Gamma, U~ = T V over T's columns 32-63 first,
      // issued as soon as they are written, then over columns 0-31
      inverse_diag32(As, Xs, Ys, TT, beta_s);
      inverse_merge64(As, Xs, Ys, TT, beta_s, [&]() {
        if (tid == 0 && alive) {
          fence_after_sync();
#pragma unroll
          for (int k16 = 2; k16 < 4; ++k16) {
            const uint64_t ad = dTTk + kstep(k16, 8192);
            mma_ss(tmem_at(tm, 0, C_W), ad, dKQm + mstep(k16), id_64x128_kmn, k16 > 2);
            mma_ss(tmem_at(tm, 0, C_U), ad, dVVm + mstep(k16), id_64x128_kmn, k16 > 2);
          }
        }
      });
      __syncthreads();
      if (tid == 0 && alive) {
        fence_after_sync();
#pragma unroll
        for (int k16 = 0; k16 < 2; ++k16) {
          const uint64_t ad = dTTk + kstep(k16, 8192);
          mma_ss(tmem_at(tm, 0, C_W), ad, dKQm + mstep(k16), id_64x128_kmn, 1);
          mma_ss(tmem_at(tm, 0, C_U), ad, dVVm + mstep(k16), id_64x128_kmn, 1);
        }
        mma_commit(bar);
        // A, X, Y consumed: G takes the log alpha of this CTA's next sub-chunk
        const int nunit = s == 0 ? unit : unit + (int)gridDim.x;
        if (nunit < a.n_units) {
          issue_la(nunit, s ^ 1);
          la_inflight = true;
        }
      }
      alive = __syncthreads_and(wait_mma(bar, phase, a.status, alive, a.wait_ns));
      fence_after_sync();
      // W -> KQ rows 0-63, U~ -> VV (fp16); M=64 accumulator layout: rows 16*sub + lane (lane < 16)
      {
        const int r = 16 * sub + lane;
        for (int cb = 0; cb < 2; ++cb) {
          const int col0 = 64 * chalf + 32 * cb;
          float w[32], u[32];
          tmem_ld32(tmem_at(tm, 32 * sub, C_W + col0), w);
          tmem_ld32(tmem_at(tm, 32 * sub, C_U + col0), u);
          tmem_wait_ld();
          if (lane < 16) {
            st_row32_h(KQ + chalf * 16384, r, col0 & 63, w);
            st_row32_h(VV + chalf * 8192, r, col0 & 63, u);
          }
        }
      }
      fence_proxy_async();
      fence_before_sync();
      __syncthreads();
      // ---------------- K~^T W, K~^T U~, P W, P U~ ----------------
      if (tid == 0 && alive) {
        fence_after_sync();
#pragma unroll
        for (int k16 = 0; k16 < 4; ++k16) {
          const uint64_t kt = dKNm + mstep(k16);
          const uint64_t wd = dKQm + mstep(k16);
          const uint64_t ud = dVVm + mstep(k16);
          const uint64_t pd = dPPk + kstep(k16, 8192);
          mma_ss(tmem_at(tm, 0, C_MK), kt, wd, id_128x128_mnmn, k16 > 0);
          mma_ss(tmem_at(tm, 0, C_BK), kt, ud, id_128x128_mnmn, k16 > 0);
          mma_ss(tmem_at(tm, 0, C_PW), pd, wd, id_64x128_kmn, k16 > 0);
          mma_ss(tmem_at(tm, 0, C_PU), pd, ud, id_64x128_kmn, k16 > 0);
        }
        mma_commit(bar);
      }
      if (tid == 0) bulk_wait_read();   // staged records read: their tiles may be rewritten
      alive = __syncthreads_and(wait_mma(bar, phase, a.status, alive, a.wait_ns));
      fence_after_sync();
      const int row = 32 * sub + lane;        // M=128 layout row
      const int r64 = 16 * sub + lane;        // M=64 layout row (lane < 16)
      if (s == 0) {
        // M_1 = Diag(Gamma_l) - K~^T W -> M1 tile;  B_1 -> B1 tile
        for (int cb = 0; cb < 2; ++cb) {
          const int col0 = 64 * chalf + 32 * cb;
          float m[32], bv[32];
          tmem_ld32(tmem_at(tm, 32 * sub, C_MK + col0), m);
          tmem_ld32(tmem_at(tm, 32 * sub, C_BK + col0), bv);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) m[j] = (row == col0 + j ? egl[row] : 0.f) - m[j];
          st_row32_h(M1 + chalf * 16384, row, col0 & 63, m);
          st_row32_h(B1 + chalf * 16384, row, col0 & 63, bv);
        }
        // R_1 = Q Gamma - P W and O'_1, staged for the record (R rows 0-63, O'' rows 0-63)
        uint8_t* stR = TT;                                  // [panel][64 rows][128 B], swizzled (TT and PP)
        uint4* stO = reinterpret_cast<uint4*>(KN);          // [c/8][64 rows][8]
        for (int cb = 0; cb < 2; ++cb) {
          const int col0 = 64 * chalf + 32 * cb;
          float pw[32], pu[32];
          tmem_ld32(tmem_at(tm, 32 * sub, C_PW + col0), pw);
          tmem_ld32(tmem_at(tm, 32 * sub, C_PU + col0), pu);
          tmem_wait_ld();
          if (lane < 16) {
            float qg[32];
            ld_row16_h(KQ + chalf * 16384, 64 + r64, col0 & 63, qg);
            ld_row16_h(KQ + chalf * 16384, 64 + r64, (col0 & 63) + 16, qg + 16);
#pragma unroll
            for (int j = 0; j < 32; ++j) qg[j] -= pw[j];
            st_row32_h(stR + chalf * 8192, r64, col0 & 63, qg);
#pragma unroll
            for (int i = 0; i < 4; ++i) stO[((col0 >> 3) + i) * 64 + r64] = pack8(pu + 8 * i);
          }
        }
        fence_proxy_async();
        fence_before_sync();
        __syncthreads();
        if (tid == 0) {
          // KQ (Q Gamma read above) and VV are free: sub-chunk 1's tiles first, then the stores
          if (alive) {
            issue_kqv(b, h, (int)t0 + SUB);
            kqv_early = true;
            kqv_inflight = true;
          }
          bulk_s2g(gR, stR, 8192);
          bulk_s2g(gR + 16384, stR + 8192, 8192);
          bulk_s2g(gO, stO, 16384);
          bulk_commit();
        }
      } else {
        // Q^_2 = Q Gamma - P W -> VV region (U~ no longer needed)
        for (int cb = 0; cb < 2; ++cb) {
          const int col0 = 64 * chalf + 32 * cb;
          float pw[32];
          tmem_ld32(tmem_at(tm, 32 * sub, C_PW + col0), pw);
          tmem_wait_ld();
          if (lane < 16) {
            float qg[32];
            ld_row16_h(KQ + chalf * 16384, 64 + r64, col0 & 63, qg);
            ld_row16_h(KQ + chalf * 16384, 64 + r64, (col0 & 63) + 16, qg + 16);
#pragma unroll
            for (int j = 0; j < 32; ++j) qg[j] -= pw[j];
            st_row32_h(VV + chalf * 8192, r64, col0 & 63, qg);
          }
        }
        __syncthreads();
        // M_2 -> KQ region (A operand, K-major, 2 panels of 16 KB)
        for (int cb = 0; cb < 2; ++cb) {
          const int col0 = 64 * chalf + 32 * cb;
          float m[32];
          tmem_ld32(tmem_at(tm, 32 * sub, C_MK + col0), m);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) m[j] = (row == col0 + j ? egl[row] : 0.f) - m[j];
          st_row32_h(KQ + chalf * 16384, row, col0 & 63, m);
        }
        fence_proxy_async();
        fence_before_sync();
        __syncthreads();
        // ---------------- combine ----------------
        if (tid == 0 && alive) {
          fence_after_sync();
          const uint32_t id_q = idesc_f16(64, 128, false, true);
#pragma unroll
          for (int k16 = 0; k16 < 8; ++k16) {
            const uint64_t m2 = dKQk + kstep(k16, 16384);
            const uint64_t q2 = dVVk + kstep(k16, 8192);
            const uint64_t m1 = dM1m + mstep(k16);
            const uint64_t b1 = dB1m + mstep(k16);
            mma_ss(tmem_at(tm, 0, C_MK), m2, m1, id_128x128_kmn, k16 > 0);   // M = M_2 M_1
            mma_ss(tmem_at(tm, 0, C_BK), m2, b1, id_128x128_kmn, 1);         // B = B_2 + M_2 B_1
            mma_ss(tmem_at(tm, 0, C_PW), q2, m1, id_q, k16 > 0);             // R_2 = Q^_2 M_1
            mma_ss(tmem_at(tm, 0, C_PU), q2, b1, id_q, 1);                   // O''_2 = O'_2 + Q^_2 B_1
          }
          mma_commit(bar);
        }
        if (tid == 0) bulk_wait_read();   // staged records read: their tiles may be rewritten
        alive = __syncthreads_and(wait_mma(bar, phase, a.status, alive, a.wait_ns));
        fence_after_sync();
        if (tid == 0 && alive) {
          // KQ and VV are free now: start the next unit's tiles before this unit's stores
          int nb_, nh_, nt0_;
          if (next_sub(unit, 1, nb_, nh_, nt0_)) {
            issue_kqv(nb_, nh_, nt0_);
            kqv_early = true;
            kqv_inflight = true;
          }
        }
        // records staged in tiles the combine products no longer read:
        //   M -> M1 region, B -> B1 region, R_2 -> TT/PP region, O''_2 -> KN region
        uint8_t* stR = TT;                               // [panel][64 rows][128 B], swizzled
        uint4* stO = reinterpret_cast<uint4*>(KN);       // [c/8][64 rows][8]
        for (int cb = 0; cb < 2; ++cb) {
          const int col0 = 64 * chalf + 32 * cb;
          float m[32], bv[32];
          tmem_ld32(tmem_at(tm, 32 * sub, C_MK + col0), m);
          tmem_ld32(tmem_at(tm, 32 * sub, C_BK + col0), bv);
          tmem_wait_ld();
          st_row32_h(M1 + chalf * 16384, row, col0 & 63, m);
          // B: [c/8][row][8]
          uint4* b16 = reinterpret_cast<uint4*>(B1);
#pragma unroll
          for (int i = 0; i < 4; ++i) b16[((col0 >> 3) + i) * 128 + row] = pack8(bv + 8 * i);
        }
        for (int cb = 0; cb < 2; ++cb) {
          const int col0 = 64 * chalf + 32 * cb;
          float rr[32], oo[32];
          tmem_ld32(tmem_at(tm, 32 * sub, C_PW + col0), rr);
          tmem_ld32(tmem_at(tm, 32 * sub, C_PU + col0), oo);
          tmem_wait_ld();
          if (lane < 16) {
            st_row32_h(stR + chalf * 8192, r64, col0 & 63, rr);
#pragma unroll
            for (int i = 0; i < 4; ++i) stO[((col0 >> 3) + i) * 64 + r64] = pack8(oo + 8 * i);
          }
        }
        fence_proxy_async();
        fence_before_sync();
        __syncthreads();
        if (tid == 0) {
          bulk_s2g(gM, M1, 32768);
          bulk_s2g(gB, B1, 32768);
          bulk_s2g(gR + 8192, stR, 8192);
          bulk_s2g(gR + 16384 + 8192, stR + 8192, 8192);
          bulk_s2g(gO + 16384, stO, 16384);
          bulk_commit();
        }
        fence_before_sync();
        __syncthreads();   // TMEM and shared tiles free for the next unit
        fence_after_sync();
      }
    }
  }
  if (tid == 0) {
    // loads still in flight after a timeout land before the CTA exits
    if (la_inflight) mbar_wait(la_bar, la_phase, 100000000ull);
    if (kqv_inflight) mbar_wait(kqv_bar, kqv_phase, 100000000ull);
    bulk_wait_all();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  if (warp == 0) tmem_dealloc(tm, 512);
}

// ---------------------------------------------------------------------------
// kda_tc_chain: per (batch item, head, CW value columns) the serial
// pass S <- M S + B over the blocks, fused with the block outputs O = R S + O''.
//   warps 0-3, the state group: thread t owns row t of S (fp32, in registers);
//     thread 0 loads M, B and issues M S.
//   warps 4-7, the output group: thread 128 + t owns token row t of the block;
//     thread 128 loads R, O'' and issues R S, off the serial path.
// Both products read the fp16 image of S_j; two images alternate so the next
// state is written while R S_j may still be reading the current one.
// ---------------------------------------------------------------------------
// Layout for CW value columns per CTA (16, 32 or 64; the MMA N is CW).
template <int CW>
struct ChainLayout {
  static constexpr int NQ = D / CW;                           // CTAs per (batch item, head)
  static constexpr uint32_t CW_BYTES = 128 * CW * 2;          // fp16 [128 rows][CW columns]
  static constexpr uint32_t SLOT = 32768 + CW_BYTES;          // 32 KB operand image + the CTA's columns of B or O''
  static constexpr uint32_t CT_O = CW;                        // TMEM: M S at column 0, R S buffers at CW and 2 CW
  static constexpr uint32_t OFF_A = 0;                        // ring A: M_j, B_j   (2 slots)
  static constexpr uint32_t OFF_B = 2 * SLOT;                 // ring B: R_j, O''_j (2 slots)
  static constexpr uint32_t OFF_S = 4 * SLOT;                 // S_j fp16 MN-major images (2 x 16 KB)
  static constexpr uint32_t OFF_BAR = OFF_S + 32768;
  static constexpr uint32_t SMEM = OFF_BAR + 256 + 1024;
};

struct ChainArgs {
  const uint8_t* ws;
  const float* S0;
  float* SN;
  __nv_bfloat16* o;
  int64_t N; int H; int n_blocks;
  uint32_t* status;
  uint64_t wait_ns;       // limit of every device wait
  int fault;              // self-test: 2 = CTA (0, 0, 0) never issues its first record load
};

// Bounded wait (at most tmo ns) that also gives up as soon as another thread of the CTA gave up.
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort_flag, uint64_t tmo) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > tmo) { *abort_flag = 1; return false; }
  }
  return true;
}

template <int CW>
__global__ void __launch_bounds__(256, 1) kda_tc_chain(ChainArgs a) {
  using L = ChainLayout<CW>;
  constexpr uint32_t CW_BYTES = L::CW_BYTES, CH_SLOT = L::SLOT, CT_O = L::CT_O;
  constexpr uint32_t CH_OFF_A = L::OFF_A, CH_OFF_B = L::OFF_B, CH_OFF_S = L::OFF_S, CH_OFF_BAR = L::OFF_BAR;
  constexpr int CK = CW < 32 ? CW : 32;   // columns per TMEM load
  constexpr uint32_t TCOLS = 3 * CW <= 64 ? 64 : (3 * CW <= 128 ? 128 : 256);   // M S and two R S buffers
  extern __shared__ uint8_t dyn[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dyn) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + CH_OFF_BAR);
  uint64_t* fullA = bars;        // [2] ring A slot landed
  uint64_t* fullB = bars + 2;    // [2] ring B slot landed
  uint64_t* msDone = bars + 4;   // M S_j complete
  uint64_t* oDone = bars + 5;    // [2] R S_j complete (TMEM buffer j&1)
  uint64_t* sReady = bars + 7;   // [2] S_j image written (128 arrivals)
  uint64_t* sFree = bars + 9;    // [2] R S_j no longer reads S image j&1
  uint64_t* oGo = bars + 11;     // [2] M S_j complete: R S_j may take the tensor pipe
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 13);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int tid = threadIdx.x, warp = tid >> 5;
  const int qtr = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int nb = a.n_blocks;
  const int64_t rec0 = ((int64_t)b * a.H + h) * nb;
  if (*(volatile uint32_t*)a.status == KDA_ERR_TIMEOUT) return;   // an earlier kernel gave up

  if (warp == 0) { tmem_alloc(tmem_slot, TCOLS); tmem_relinquish(); }
  if (tid == 0) {
    for (int i = 0; i < 13; ++i) mbar_init(&bars[i], (i == 7 || i == 8) ? 128 : 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tm = *tmem_slot;
  const uint32_t idesc = idesc_f16(128, CW, false, true);
  const uint64_t dS = mdesc0(smem_u32(sm + CH_OFF_S), 16384);
  const int lane_base = 32 * (warp & 3);
  bool ok = true;

  if (warp < 4) {
    // ---------------- state group ----------------
    const int row = tid;
    auto load_A = [&](int j) {
      uint8_t* dst = sm + CH_OFF_A + (j & 1) * CH_SLOT;
      const uint8_t* rec = a.ws + (rec0 + j) * kBlockBytes;
      mbar_arrive_expect_tx(&fullA[j & 1], CH_SLOT);
      bulk_g2s(dst, rec + kMOff, 32768, &fullA[j & 1]);
      bulk_g2s(dst + 32768, rec + kBOff + qtr * CW_BYTES, CW_BYTES, &fullA[j & 1]);
    };
    // thread 32 refills ring A, so thread 0 goes from the barrier straight to the next product
    const bool loaderA = tid == 32;
    // self-test of the bounded waits: the first record load is never issued, so its wait gives up
    const bool skipA0 = a.fault == 2 && qtr == 0 && h == 0 && b == 0;
    int issuedA = 0, mma_pending = 0;
    if (loaderA)
      for (; issuedA < 2 && issuedA < nb; ++issuedA)
        if (!(skipA0 && issuedA == 0)) load_A(issuedA);
    float S[CW];
#pragma unroll
    for (int c = 0; c < CW; ++c)
      S[c] = a.S0 ? a.S0[(((int64_t)b * a.H + h) * D + row) * D + CW * qtr + c] : 0.f;
    auto store_S = [&](int slot) {
      uint8_t* img = sm + CH_OFF_S + slot * 16384;
#pragma unroll
      for (int i = 0; i < CW / 8; ++i) *reinterpret_cast<uint4*>(img + swz_off(row, 8 * i)) = pack8(S + 8 * i);
      fence_proxy_async();
      mbar_arrive(&sReady[slot]);
    };
    store_S(0);
    ok = named_sync_and(1, 128, ok);
    const uint64_t dA = kdesc0(smem_u32(sm + CH_OFF_A));
    int j = 0;
    for (; j < nb && ok; ++j) {
      if (tid == 0) {
        const bool landed = wait_or_abort(&fullA[j & 1], (uint32_t)(j >> 1) & 1u, abort_flag, a.wait_ns);
        if (landed) {
          fence_after_sync();
          const uint64_t da = dA + (uint32_t)(j & 1) * (CH_SLOT >> 4);
          const uint64_t db = dS + (uint32_t)(j & 1) * (16384u >> 4);
#pragma unroll
          for (int k16 = 0; k16 < 8; ++k16) mma_ss(tm, da + kstep(k16, 16384), db + mstep(k16), idesc, k16 > 0);
          mma_commit(msDone);
          mma_commit(&oGo[j & 1]);
          mma_pending = 1;
        }
      }
      bool mine = wait_or_abort(msDone, (uint32_t)j & 1u, abort_flag, a.wait_ns);
      if (tid == 0 && mine) mma_pending = 0;
      mine = mine && wait_or_abort(&fullA[j & 1], (uint32_t)(j >> 1) & 1u, abort_flag, a.wait_ns);   // B_j visible here too
      if (mine) {
        fence_after_sync();
        const uint4* Bs = reinterpret_cast<const uint4*>(sm + CH_OFF_A + (j & 1) * CH_SLOT + 32768);
#pragma unroll
        for (int c0 = 0; c0 < CW; c0 += CK) {
          float v[CK];
          tmem_ld_n(tmem_at(tm, lane_base, c0), v);
          uint4 bu[CK / 8];
#pragma unroll
          for (int i = 0; i < CK / 8; ++i) bu[i] = Bs[((c0 >> 3) + i) * 128 + row];
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < CK / 8; ++i) {
            float bf[8];
            unpack8(bu[i], bf);
#pragma unroll
            for (int e = 0; e < 8; ++e) S[c0 + 8 * i + e] = v[8 * i + e] + bf[e];
          }
        }
        if (j + 1 < nb) {
          // image (j+1)&1 last held S_{j-1}; R S_{j-1} must be done with it
          if (j >= 1) mine = wait_or_abort(&sFree[(j - 1) & 1], (uint32_t)((j - 1) >> 1) & 1u, abort_flag, a.wait_ns);
          if (mine) store_S((j + 1) & 1);
        }
      }
      fence_before_sync();
      ok = named_sync_and(1, 128, mine);   // ring A slot j consumed, S_{j+1} image written
      if (ok && loaderA && issuedA < nb) { load_A(issuedA); ++issuedA; }
    }
    if (ok && a.SN) {
#pragma unroll
      for (int c = 0; c < CW; ++c) a.SN[(((int64_t)b * a.H + h) * D + row) * D + CW * qtr + c] = S[c];
    }
    if (tid == 0 && mma_pending) mbar_wait(msDone, (uint32_t)(j - 1) & 1u, 100000000ull);
    if (loaderA)   // each slot's latest load lands before the CTA exits (consumed ones return at once)
      for (int jj = max(0, issuedA - 2); jj < issuedA; ++jj)
        if (!(skipA0 && jj == 0)) mbar_wait(&fullA[jj & 1], (uint32_t)(jj >> 1) & 1u, 100000000ull);
  } else {
    // ---------------- output group ----------------
    const int r = tid - 128;   // token row of the block = TMEM lane
    const bool leader = r == 0;
    auto load_B = [&](int j) {
      uint8_t* dst = sm + CH_OFF_B + (j & 1) * CH_SLOT;
      const uint8_t* rec = a.ws + (rec0 + j) * kBlockBytes;
      mbar_arrive_expect_tx(&fullB[j & 1], CH_SLOT);
      bulk_g2s(dst, rec + kROff, 32768, &fullB[j & 1]);
      bulk_g2s(dst + 32768, rec + kOOff + qtr * (CW_BYTES / 2), CW_BYTES / 2, &fullB[j & 1]);
      bulk_g2s(dst + 32768 + CW_BYTES / 2, rec + kOOff + 16384 + qtr * (CW_BYTES / 2), CW_BYTES / 2, &fullB[j & 1]);
    };
    // thread 160 refills ring B, so the leader goes from the barrier straight to the next product
    const bool loaderB = r == 32;
    int issuedB = 0, o_pending = -1;
    if (loaderB)
      for (; issuedB < 2 && issuedB < nb; ++issuedB) load_B(issuedB);
    const uint64_t dR = kdesc0(smem_u32(sm + CH_OFF_B));
    const int64_t tok_stride = (int64_t)a.H * D;
    __nv_bfloat16* obase = a.o + (int64_t)b * a.N * tok_stride + (int64_t)h * D + CW * qtr;
    for (int j = 0; j < nb && ok; ++j) {
      if (leader) {
        bool go = wait_or_abort(&sReady[j & 1], (uint32_t)(j >> 1) & 1u, abort_flag, a.wait_ns);
        // issued once M S_j is done, so it does not share the tensor pipe with the serial product
        go = go && wait_or_abort(&oGo[j & 1], (uint32_t)(j >> 1) & 1u, abort_flag, a.wait_ns);
        go = go && wait_or_abort(&fullB[j & 1], (uint32_t)(j >> 1) & 1u, abort_flag, a.wait_ns);
        if (go) {
          fence_after_sync();
          const uint64_t da = dR + (uint32_t)(j & 1) * (CH_SLOT >> 4);
          const uint64_t db = dS + (uint32_t)(j & 1) * (16384u >> 4);
          const uint32_t d = tm + CT_O + CW * (uint32_t)(j & 1);
#pragma unroll
          for (int k16 = 0; k16 < 8; ++k16) mma_ss(d, da + kstep(k16, 16384), db + mstep(k16), idesc, k16 > 0);
          mma_commit(&oDone[j & 1]);
          mma_commit(&sFree[j & 1]);
          o_pending = j;
        }
      }
      bool mine = wait_or_abort(&oDone[j & 1], (uint32_t)(j >> 1) & 1u, abort_flag, a.wait_ns);
      if (leader && mine) o_pending = -1;
      mine = mine && wait_or_abort(&fullB[j & 1], (uint32_t)(j >> 1) & 1u, abort_flag, a.wait_ns);   // O''_j visible here too
      if (mine) {
        fence_after_sync();
        const uint4* Oo = reinterpret_cast<const uint4*>(sm + CH_OFF_B + (j & 1) * CH_SLOT + 32768);
        const int64_t tok = (int64_t)j * BLK + r;
        __nv_bfloat16* orow = obase + tok * tok_stride;
#pragma unroll
        for (int c0 = 0; c0 < CW; c0 += CK) {
          float v[CK];
          tmem_ld_n(tmem_at(tm, lane_base, CT_O + CW * (j & 1) + c0), v);
          uint4 ou[CK / 8];
#pragma unroll
          for (int i = 0; i < CK / 8; ++i) ou[i] = Oo[((r >> 6) * (CW / 8) + (c0 >> 3) + i) * 64 + (r & 63)];
          tmem_wait_ld();
          if (tok < a.N) {
#pragma unroll
            for (int i = 0; i < CK / 8; ++i) {
              float of[8];
              unpack8(ou[i], of);
              uint32_t w[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                __nv_bfloat162 hh = __floats2bfloat162_rn(v[8 * i + 2 * e] + of[2 * e], v[8 * i + 2 * e + 1] + of[2 * e + 1]);
                w[e] = *reinterpret_cast<uint32_t*>(&hh);
              }
              reinterpret_cast<uint4*>(orow + c0)[i] = make_uint4(w[0], w[1], w[2], w[3]);
            }
          }
        }
      }
      fence_before_sync();
      ok = named_sync_and(2, 128, mine);   // TMEM buffer j&1 read, ring B slot j consumed
      if (ok && loaderB && issuedB < nb) { load_B(issuedB); ++issuedB; }
    }
    if (leader && o_pending >= 0) mbar_wait(&oDone[o_pending & 1], (uint32_t)(o_pending >> 1) & 1u, 100000000ull);
    if (loaderB)
      for (int jj = max(0, issuedB - 2); jj < issuedB; ++jj)
        mbar_wait(&fullB[jj & 1], (uint32_t)(jj >> 1) & 1u, 100000000ull);
  }
  if (tid == 0 && *abort_flag) set_status(a.status, KDA_ERR_TIMEOUT);
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  if (warp == 0) tmem_dealloc(tm, TCOLS);
}

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// [B][N][H][128] activations seen as a 4D tensor (channel, head, token, item);
// box: box_c channels x 1 head x 64 tokens x 1 item.  Tokens past N read as zero.
bool encode_act_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int es, const Dims& d, int box_c,
                    bool swizzle128) {
  const PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)d.H, (cuuint64_t)d.N, (cuuint64_t)d.B};
  const cuuint64_t strides[3] = {(cuuint64_t)D * es, (cuuint64_t)d.H * D * es, (cuuint64_t)d.N * d.H * D * es};
  const cuuint32_t box[4] = {(cuuint32_t)box_c, 1u, (cuuint32_t)SUB, 1u};
  const cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  return enc(m, dt, 4, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int CW>
cudaError_t launch_chain(const ChainArgs& ca, dim3 grid, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(kda_tc_chain<CW>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)ChainLayout<CW>::SMEM);
  if (e != cudaSuccess) return e;
  kda_tc_chain<CW><<<grid, 256, ChainLayout<CW>::SMEM, s>>>(ca);
  return cudaGetLastError();
}

template <typename TIn>
cudaError_t launch_all(const Dims& d, const void* q, const void* k, const void* v, const float* la,
                       const void* beta, const float* S0, void* o, float* SN, uint8_t* ws, uint32_t* status,
                       cudaStream_t s, int* launches, int fault, uint64_t wait_ns) {
  const int n_blocks = (int)((d.N + BLK - 1) / BLK);
  cudaError_t e;
  int dev = 0, n_sm = 148;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  e = cudaFuncSetAttribute(kda_tc_prep<TIn>, cudaFuncAttributeMaxDynamicSharedMemorySize, PREP_SMEM);
  if (e != cudaSuccess) return e;

  const int BH = d.B * d.H;
  const int n_units = BH * n_blocks;
  PrepArgs pa{q, k, v, la, beta, ws, d.N, d.H, BH, n_blocks, n_units, status, wait_ns, fault};
  PrepMaps mp;
  const CUtensorMapDataType adt = kIsHalf<TIn> ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if (!encode_act_map(&mp.q, q, adt, 2, d, 64, true) || !encode_act_map(&mp.k, k, adt, 2, d, 64, true) ||
      !encode_act_map(&mp.v, v, adt, 2, d, 64, true) ||
      !encode_act_map(&mp.la, la, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, d, 128, false))
    return cudaErrorInvalidValue;
  // the records depend on q, k, v, log alpha and beta only: a caller that kept them (same inputs,
  // same workspace) runs the state pass alone
  if (!d.reuse_records) {
    kda_tc_prep<TIn><<<dim3((unsigned)min(n_units, n_sm)), 256, PREP_SMEM, s>>>(pa, mp);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  ChainArgs ca{ws, S0, SN, static_cast<__nv_bfloat16*>(o), d.N, d.H, n_blocks, status, wait_ns, fault};
  // the narrowest column split whose grid fits on the SMs (the serial pass is latency bound)
  const int bh = d.B * d.H;
  if (ChainLayout<16>::NQ * bh <= n_sm) e = launch_chain<16>(ca, dim3(ChainLayout<16>::NQ, d.H, d.B), s);
  else if (ChainLayout<32>::NQ * bh <= n_sm) e = launch_chain<32>(ca, dim3(ChainLayout<32>::NQ, d.H, d.B), s);
  else e = launch_chain<64>(ca, dim3(ChainLayout<64>::NQ, d.H, d.B), s);
  if (e != cudaSuccess) return e;
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (launches) *launches += d.reuse_records ? 1 : 2;
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
                            void* ws, uint32_t* status, cudaStream_t s, int* launches, int fault,
                            uint64_t wait_ns) {
  // beta and o are bf16 (the problem dtype); q', k', v' are fp16 (internal conv output) or bf16 (caller)
  if (in_f16)
    return launch_all<__half>(d, q, k, v, log_alpha, beta, S0, o, SN, static_cast<uint8_t*>(ws), status, s,
                              launches, fault, wait_ns);
  return launch_all<__nv_bfloat16>(d, q, k, v, log_alpha, beta, S0, o, SN, static_cast<uint8_t*>(ws), status, s,
                                   launches, fault, wait_ns);
}

}  // namespace kda
