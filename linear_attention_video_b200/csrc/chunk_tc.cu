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
//                 record per unit (M, B, R, O'' in fp16 operand images).  With few
//                 (batch item, head) pairs it is a cooperative launch whose first
//                 CTAs, one per pair, run the serial pass S <- M S + B and the block
//                 outputs O = R S + O'' as the other CTAs publish the records.
//   kda_tc_chain  one CTA per (batch item, head, 16, 32 or 64 value columns):
//                 the serial pass and the outputs over records already written
//                 (records kept from an earlier call, or many pairs).
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
//   R   MN-major operand image: 2 token panels [128 channels][64 tokens]   32 KB
//   O'' [token half][128 channels][64 tokens], 128-byte-swizzled rows   32 KB
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
// KK and VV adjacent: W^T and U~^T form one [256][64] K-major operand (N = 256 products);
// QQ and KN adjacent: M_2 ([128][128], two 16 KB panels) for the combine
constexpr uint32_t OFF_KK = 0;          // [64][128] fp16: K Gamma, then W^T ([128 channels][64 tokens]), then -Q^_2
constexpr uint32_t OFF_VV = 16384;      // [64][128] fp16: V (TMA), then U~^T ([128 channels][64 tokens])
constexpr uint32_t OFF_QQ = 32768;      // [64][128] fp16: Q Gamma; with KN: M_2
constexpr uint32_t OFF_KN = 49152;      // [64][128] fp16: K~; staging of O'_1 and O''_2
constexpr uint32_t OFF_TT = 65536;      // [64][64] fp16: T, then the identity (TT and PP together: staging of R_1, R_2)
constexpr uint32_t OFF_PP = 73728;      // [64][64] fp16: P
constexpr uint32_t OFF_M1 = 81920;      // [128][128] fp16: M_1 (MN-major operand image)
constexpr uint32_t OFF_B1 = 114688;     // [128][128] fp16: B_1 (MN-major operand image)
// 72 KB used three ways in turn: the inputs of a sub-chunk (TMA targets: log alpha [64 tokens][128] fp32,
// raw k and q at G_IN), the operand tiles of the Gram, and A, X, Y of the blocked inverse
constexpr uint32_t OFF_G = 147456;
constexpr uint32_t G_IN = 32768;        // raw k (rows 0-63) and q (rows 64-127): 2 panels [128][64] of 16 KB
constexpr uint32_t G_ROW = 0;           // level tiles, rows: [64][128] fp16 per level (5, 4, 3), 16 KB apart
constexpr uint32_t G_COL = 49152;       // level tiles, columns: [32][128] fp16 per level, 8 KB apart
constexpr uint32_t G_DCOL = 32768;      // direct Gram: rows [128][128] at G_ROW, columns [64][128] here
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
// direct Gram factorisation (e^{g_r - g_31} e^{g_31 - g_i}) only while every fp16 factor stays small:
// the decay over each half of the sub-chunk at most kHalfRange nats, |k|, |q| at most kMagRange
// (operands then stay below kMagRange e^kHalfRange = 25,800, inside fp16)
constexpr float kHalfRange = 6.f;
constexpr float kMagRange = 64.f;

// TMEM columns
constexpr int C_G = 0;                   // the three Gram levels, 32 columns each (M = 64 layout)
constexpr int C_W = 128, C_U = 192;      // W^T, U~^T: M = 128 (channels) x 64 tokens
constexpr int C_MK = 0, C_BK = 128;        // M = 128 x 128 each
constexpr int C_RT = 256, C_OT = 320;      // R^T, O'^T (and the combine's R_2^T, O''_2^T): M = 128 x 64

// TMA descriptors of the [B][N][H][128] inputs, box [1][64 tokens][1][64 or 128 channels]
struct PrepMaps {
  CUtensorMap q, k, v;   // 64-channel boxes, 128-byte swizzle: one operand panel each
  CUtensorMap la;        // 128-channel box, no swizzle
  CUtensorMap o;         // output (bf16), 64-channel boxes, 128-byte swizzle: stores of the state role
};

struct PrepArgs {
  const void* q; const void* k; const void* v;
  const float* la; const void* beta;
  uint8_t* ws;            // block records
  int64_t N; int H; int BH; int n_blocks; int n_units;
  uint32_t* status;
  uint64_t wait_ns;       // limit of every device wait
  int fault;              // self-test: 1 = the first record CTA never issues its first k/q/v load;
                          //            2 = the state CTA of (0, 0) never issues its first record load
  // with n_state > 0, CTAs 0 .. n_state-1 run the state pass (one per batch item and head) beside
  // the record CTAs: a record CTA publishes each finished record by writing `token` to its flag
  int n_state;
  uint32_t* flags;        // [B][H][n_blocks]
  uint32_t token;
  const float* S0; float* SN; __nv_bfloat16* o;
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

// Named barrier over `count` threads (a multiple of 32) on hardware barrier `id` (1..15).
__device__ __forceinline__ void named_sync(uint32_t id, uint32_t count) {
  asm volatile("bar.sync %0, %1;" :: "r"(id), "r"(count) : "memory");
}

// Blocked inverse X = (I + A)^{-1} of the unit lower-triangular 64x64 matrix, A strictly
// lower in As, delivered as T = X Diag(beta) in fp16 (TT, one swizzled K-major panel).
// Warps 0-3 compute; warps 4-7 write the zero blocks of T above the diagonal blocks.
//   1. warp w: diagonal 16x16 block D_w by forward substitution (lane = column, lanes 0-15);
//      lanes 16-31 of warps 0 and 2 zero the blocks of X above D_0 and D_2 that step 3 reads.
//   2. pairs (0, 1) and (2, 3): the diagonal 32x32 blocks, X_10 = -D_1 (A_10 D_0); each warp of
//      the pair one 8-column tile of both products.
//   3. warps 0-3: X_21 = -X_22 (A_21 X_11) of the 64x64 matrix; warp w the 8-column tile w of
//      both products (32 rows).
// The products run on the warp-level tensor cores in tf32 with split operands (about fp32
// accuracy).  A tile's partial product Y goes through warp-private shared memory: a column
// tile of the result needs only the same column tile of Y, so steps 2 and 3 synchronise only
// the warps that produce their inputs (named barriers 1-3).  The caller's next barrier
// publishes T.
__device__ void inverse64(const float* As, float* Xs, float* Ys, uint8_t* TT, const float* beta) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t4 = lane & 3;
  auto st_t = [&](int r, int c, float v0, float v1) {   // T[r][c], T[r][c + 1] (c even)
    st_h2(TT + swz_off(r, c), v0 * beta[c], v1 * beta[c + 1]);
  };
  if (warp >= 4) {
    // 8-column chunks of T above the diagonal blocks: rows 0-15 chunks 2-7, rows 16-31 chunks 4-7,
    // rows 32-47 chunks 6-7
    for (int e = tid - 128; e < 192; e += 128) {
      int r, c8;
      if (e < 96) { r = e / 6; c8 = 2 + e % 6; }
      else if (e < 160) { r = 16 + (e - 96) / 4; c8 = 4 + (e - 96) % 4; }
      else { r = 32 + (e - 160) / 2; c8 = 6 + (e - 160) % 2; }
      *reinterpret_cast<uint4*>(TT + swz_off(r, 8 * c8)) = make_uint4(0u, 0u, 0u, 0u);
    }
    fence_proxy_async();
    return;
  }
  float* Yw = Ys + warp * 256;   // warp-private scratch, [16 or 32 rows][8]
  {
    // 1. diagonal block `warp`
    const int o = 16 * warp;
    if (lane < 16) {
      const int l = lane;
      float x[16];
#pragma unroll
      for (int r = 0; r < 16; ++r) x[r] = r == l ? 1.f : 0.f;
      // row r: x[r] -= A[r][m] x[m] for m = 0 .. r-1, A's row read 4 wide
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
      const float bl = beta[o + l];
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        Xs[(o + r) * LDXS + o + l] = x[r];
        *reinterpret_cast<__half*>(TT + swz_off(o + r, o + l)) = __float2half_rn(x[r] * bl);
      }
    } else if ((warp & 1) == 0) {
      // zero block of X above D_0 (rows 0-15, columns 16-31) or D_2 (rows 32-47, columns 48-63)
      const int l = lane - 16;
#pragma unroll
      for (int r = 0; r < 16; ++r) Xs[(o + r) * LDXS + o + 16 + l] = 0.f;
    }
  }
  named_sync(1 + (warp >> 1), 64);   // D_0, D_1 (or D_2, D_3) in place
  {
    // 2. 32x32 merge of pair p, column tile nt: X_10[:, nt] = -D_1 (A_10 D_0[:, nt])
    const int p = warp >> 1, nt = warp & 1, o = 32 * p;
    float d[4];
    mma_tile_3xtf32(As + (o + 16) * LDA + o, LDA, Xs + o * LDXS + o + 8 * nt, LDXS, 2, g, t4, d);
    Yw[g * 8 + 2 * t4] = d[0];
    Yw[g * 8 + 2 * t4 + 1] = d[1];
    Yw[(g + 8) * 8 + 2 * t4] = d[2];
    Yw[(g + 8) * 8 + 2 * t4 + 1] = d[3];
    __syncwarp();
    mma_tile_3xtf32(Xs + (o + 16) * LDXS + o + 16, LDXS, Yw, 8, 2, g, t4, d);
    const int r0 = o + 16 + g, c = o + 8 * nt + 2 * t4;
    Xs[r0 * LDXS + c] = -d[0];
    Xs[r0 * LDXS + c + 1] = -d[1];
    Xs[(r0 + 8) * LDXS + c] = -d[2];
    Xs[(r0 + 8) * LDXS + c + 1] = -d[3];
    st_t(r0, c, -d[0], -d[1]);
    st_t(r0 + 8, c, -d[2], -d[3]);
  }
  named_sync(3, 128);   // X_11 and X_22 in place
  {
    // 3. 64x64 merge, column tile `warp` of X_21 = -X_22 (A_21 X_11), rows 32-63
    const int c0 = 8 * warp;
    float d0[4], d1[4];
    mma_tile_3xtf32(As + 32 * LDA, LDA, Xs + c0, LDXS, 4, g, t4, d0);   // rows 32-47 of A_21 X_11
    mma_tile_3xtf32(As + 48 * LDA, LDA, Xs + c0, LDXS, 4, g, t4, d1);   // rows 48-63
    __syncwarp();   // step 2's reads of the scratch are done
    Yw[g * 8 + 2 * t4] = d0[0];
    Yw[g * 8 + 2 * t4 + 1] = d0[1];
    Yw[(g + 8) * 8 + 2 * t4] = d0[2];
    Yw[(g + 8) * 8 + 2 * t4 + 1] = d0[3];
    Yw[(g + 16) * 8 + 2 * t4] = d1[0];
    Yw[(g + 16) * 8 + 2 * t4 + 1] = d1[1];
    Yw[(g + 24) * 8 + 2 * t4] = d1[2];
    Yw[(g + 24) * 8 + 2 * t4 + 1] = d1[3];
    __syncwarp();
    mma_tile_3xtf32(Xs + 32 * LDXS + 32, LDXS, Yw, 8, 4, g, t4, d0);   // X_22 rows 32-47 times Y
    mma_tile_3xtf32(Xs + 48 * LDXS + 32, LDXS, Yw, 8, 4, g, t4, d1);   // rows 48-63
    const int c = c0 + 2 * t4;
    st_t(32 + g, c, -d0[0], -d0[1]);
    st_t(40 + g, c, -d0[2], -d0[3]);
    st_t(48 + g, c, -d1[0], -d1[1]);
    st_t(56 + g, c, -d1[2], -d1[3]);
  }
  fence_proxy_async();
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

// Two fp32 values in one 64-bit register pair, for the packed fp32x2 multiply of sm_100.
__device__ __forceinline__ uint64_t f2pack(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ float2 f2unpack(uint64_t v) {
  float a, b;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
  return make_float2(a, b);
}
__device__ __forceinline__ uint64_t f2mul(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
// 4 fp16 at p from two packed fp32 pairs
__device__ __forceinline__ void st_h4x2(uint8_t* p, uint64_t lo, uint64_t hi) {
  const float2 a = f2unpack(lo), b = f2unpack(hi);
  st_h4(p, a.x, a.y, b.x, b.y);
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

// ---------------------------------------------------------------------------
// State role (CTAs 0 .. n_state-1 of a launch that has them): for one (batch item, head),
// block by block as the record CTAs publish them,
//   S_{j+1} = M_j S_j + B_j   and   O_j = R_j S_j + O''_j,
// on the tensor core at the full 128-column width of S.
//   warps 0-3, the state group: thread 0 issues M_j S_j; row k = tid of S (TMEM lane k) adds B_j
//     (read from L2 into registers while the product runs) and writes the fp16 image of S_{j+1},
//     the MN-major B operand of the next block's products.  This is the serial part.
//   warps 4-7, the output group: thread 128 issues R_j S_j and then O''_j I (the identity adds
//     O'' in the accumulator) into one of two TMEM buffers; token row r = tid - 128 (TMEM lane r)
//     converts O_j to bf16 and stages it; thread 128 stores the staged rows by TMA.
// M_{j+1}, R_{j+1} and O''_{j+1} are loaded as soon as the product that read the slot is
// complete.  Records are read only after their flags are acquired: a lead thread reads the
// flags of up to eight blocks ahead with relaxed loads and acquires those published, in order,
// with one fence; the loads then cross into the async proxy.
// ---------------------------------------------------------------------------
constexpr uint32_t ST_S = 0, ST_M = 32768, ST_R = 65536, ST_O = 98304, ST_I = 131072, ST_STG = 163840,
                   ST_BAR = 196608;
constexpr int ST_TS = 0, ST_TO = 128;   // TMEM: S at columns 0-127, O in two buffers at 128 and 256

// Acquires the flags of blocks ready, ready + 1, ... (up to eight per poll) until block `need`
// is acquired; at most tmo ns, less if another CTA recorded a timeout.
__device__ __forceinline__ bool acquire_through(const uint32_t* flags, int need, int nb, int& ready, uint32_t token,
                                                uint32_t* status, uint64_t tmo) {
  if (need < ready) return true;
  uint64_t t0 = 0;
  for (;;) {
    const int n_poll = min(8, nb - ready);
    uint32_t f[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) f[i] = i < n_poll ? ld_relaxed_gpu(flags + ready + i) : 0u;
    int n = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) n += (n == i && f[i] == token) ? 1 : 0;   // published prefix
    if (n > 0) {
      fence_acq_rel_gpu();   // the relaxed reads that saw the releases become acquires
      ready += n;
      if (need < ready) return true;
      continue;
    }
    if (t0 == 0) t0 = globaltimer_ns();
    if (*(volatile uint32_t*)status == KDA_ERR_TIMEOUT) return false;
    if (globaltimer_ns() - t0 > tmo) { set_status(status, KDA_ERR_TIMEOUT); return false; }
    __nanosleep(64);
  }
}

// Bounded mbarrier wait that also gives up once another thread of the CTA gave up.
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort_flag, uint64_t tmo) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > tmo) { *abort_flag = 1; return false; }
  }
  return true;
}

__device__ __noinline__ void state_role(const PrepArgs& a, const CUtensorMap* o_map, uint8_t* sm) {
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + ST_BAR);
  uint64_t* m_full = bars;           // record parts landed
  uint64_t* r_full = bars + 1;
  uint64_t* o_full = bars + 2;
  uint64_t* ms_issued = bars + 3;    // M_j S_j is in the tensor pipe (R_j S_j goes after it)
  uint64_t* ms_done = bars + 4;      // M_j S_j complete
  uint64_t* rs_done = bars + 5;      // R_j S_j complete: S_j and R_j no longer read
  uint64_t* od_done = bars + 6;      // O''_j I complete: O_j in TMEM, O''_j no longer read
  uint64_t* fin = bars + 7;          // [2] every product of thread 0 / 128 complete (exit path)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 9);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int tid = threadIdx.x, warp = tid >> 5;
  const int bh = (int)blockIdx.x, b = bh / a.H, h = bh - b * a.H;
  const int nb = a.n_blocks;
  const int64_t rec0 = (int64_t)bh * nb;
  const uint64_t tmo = a.wait_ns;
  const uint32_t* flags = a.flags + rec0;
  const uint64_t pol_once = l2_policy_evict_first();   // each record part is read once
  auto rec = [&](int j) { return a.ws + (rec0 + j) * kBlockBytes; };
  if (warp == 0) { tmem_alloc(tmem_slot, 512); tmem_relinquish(); }
  if (tid == 0) {
    for (int i = 0; i < 9; ++i) mbar_init(&bars[i], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  // fp16 images, rows 0-127 at (panel n / 64, row, column n % 64): S_0 (threads 0-127) and the
  // identity (threads 128-255)
  {
    const int row = tid & 127;
    const float* s0 = (tid < 128 && a.S0) ? a.S0 + ((int64_t)bh * D + row) * D : nullptr;
#pragma unroll
    for (int n0 = 0; n0 < D; n0 += 32) {
      float v[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) v[e] = tid < 128 ? (s0 ? s0[n0 + e] : 0.f) : (row == n0 + e ? 1.f : 0.f);
      st_row32_h(sm + (tid < 128 ? ST_S : ST_I) + (n0 >> 6) * 16384, row, n0 & 63, v);
    }
  }
  fence_proxy_async();
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tm = *tmem_slot;
  const int lane_base = 32 * (warp & 3);
  const uint64_t dS = mdesc0(smem_u32(sm + ST_S), 16384);     // S_j: MN-major, two column panels
  bool ok = true;

  if (warp < 4) {
    // ---------------- state group ----------------
    const int k = tid;
    const bool lead = tid == 0;
    const uint64_t dM = kdesc0(smem_u32(sm + ST_M));            // M_j: K-major, two 16 KB K-panels
    const uint32_t id_ms = idesc_f16(128, 128, false, true);
    int m_in = -1;          // lead: block of a load issued and not yet waited for
    bool issued = false;    // lead: some product was issued
    int ready = 0;          // lead: flags of blocks < ready acquired
    // self-test of the bounded waits: the first record load of (0, 0) is never issued
    const bool skip0 = a.fault == 2 && bh == 0;
    if (lead) {
      ok = acquire_through(flags, 0, nb, ready, a.token, a.status, tmo);
      if (ok && !skip0) {
        fence_proxy_async_global();
        mbar_arrive_expect_tx(m_full, 32768);
        bulk_g2s_hint(sm + ST_M, rec(0) + kMOff, 32768, m_full, pol_once);
        m_in = 0;
      }
      if (!ok) *abort_flag = 1;
    }
    ok = named_sync_and(1, 128, ok);   // also orders the B loads below after the lead's acquire
    int j = 0;
    for (; j < nb && ok; ++j) {
      const uint32_t par = (uint32_t)j & 1u;
      // B_j row k from L2 into registers while M_j S_j runs ([c/8][row][8]; not cached in L1)
      uint4 bu[16];
      {
        const uint4* Bg = reinterpret_cast<const uint4*>(rec(j) + kBOff);
#pragma unroll
        for (int i = 0; i < 16; ++i) bu[i] = __ldcg(Bg + i * 128 + k);
      }
      bool mine = true;
      if (lead) {
        // M_j S_j as soon as M_j has landed (the image of S_j was written before the last barrier)
        mine = wait_or_abort(m_full, par, abort_flag, tmo);
        if (mine) {
          m_in = -1;
          fence_after_sync();
#pragma unroll
          for (int k16 = 0; k16 < 8; ++k16)
            mma_ss(tmem_at(tm, 0, ST_TS), dM + kstep(k16, 16384), dS + mstep(k16), id_ms, k16 > 0);
          mma_commit(ms_done);
          issued = true;
          mbar_arrive(ms_issued);
          // the next record's flag, while the product runs
          if (j + 1 < nb) mine = acquire_through(flags, j + 1, nb, ready, a.token, a.status, tmo);
        }
        if (!mine) *abort_flag = 1;
      }
      mine = mine && wait_or_abort(ms_done, par, abort_flag, tmo);
      if (lead && mine && j + 1 < nb) {   // M_j is consumed: M_{j+1} next
        fence_proxy_async_global();
        mbar_arrive_expect_tx(m_full, 32768);
        bulk_g2s_hint(sm + ST_M, rec(j + 1) + kMOff, 32768, m_full, pol_once);
        m_in = j + 1;
      }
      if (mine) {
        fence_after_sync();
        float* sn = (j + 1 == nb && a.SN) ? a.SN + ((int64_t)bh * D + k) * D : nullptr;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          float sv[64];
          tmem_ld32(tmem_at(tm, lane_base, ST_TS + 64 * half), *reinterpret_cast<float(*)[32]>(sv));
          tmem_ld32(tmem_at(tm, lane_base, ST_TS + 64 * half + 32), *reinterpret_cast<float(*)[32]>(sv + 32));
          tmem_wait_ld();
          uint4 pk[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            float bf[8];
            unpack8(bu[8 * half + i], bf);
#pragma unroll
            for (int e = 0; e < 8; ++e) sv[8 * i + e] += bf[e];
            pk[i] = pack8(sv + 8 * i);
          }
          if (sn) {   // the final state, fp32
#pragma unroll
            for (int i = 0; i < 16; ++i)
              reinterpret_cast<float4*>(sn + 64 * half)[i] = make_float4(sv[4 * i], sv[4 * i + 1], sv[4 * i + 2], sv[4 * i + 3]);
          }
          // S_j is read by R_j S_j too: its image is rewritten only after that product
          if (half == 0) mine = wait_or_abort(rs_done, par, abort_flag, tmo);
          if (mine) {
#pragma unroll
            for (int i = 0; i < 8; ++i) *reinterpret_cast<uint4*>(sm + ST_S + half * 16384 + swz_off(k, 8 * i)) = pk[i];
          }
        }
      }
      fence_proxy_async();   // the image of S_{j+1}, read next by the tensor core
      fence_before_sync();
      ok = named_sync_and(1, 128, mine);   // S_{j+1} written; S TMEM read; flag j+1 acquired
      fence_after_sync();
    }
    if (lead) {
      // work in flight after a timeout finishes before the CTA frees its memory
      if (issued) {
        mma_commit(&fin[0]);   // arrives once every product this thread issued is complete
        mbar_wait(&fin[0], 0u, 100000000ull);
      }
      // a slot's pending load is its latest: the earlier phases of its barrier were all waited for
      if (m_in >= 0) mbar_wait(m_full, (uint32_t)m_in & 1u, 100000000ull);
    }
  } else {
    // ---------------- output group ----------------
    const int r = tid - 128;
    const bool lead = r == 0;
    const uint64_t dR = mdesc0(smem_u32(sm + ST_R), 16384);     // R_j: MN-major, two token panels
    const uint64_t dO = mdesc0(smem_u32(sm + ST_O), 16384);     // O''_j: MN-major, two token panels
    const uint64_t dI = mdesc0(smem_u32(sm + ST_I), 16384);
    const uint32_t id_mn = idesc_f16(128, 128, true, true);
    int r_in = -1, o_in = -1;   // lead: block of a load issued and not yet waited for
    bool issued = false;
    int ready = 0;              // lead: flags of blocks < ready acquired
    if (lead) {
      ok = acquire_through(flags, 0, nb, ready, a.token, a.status, tmo);
      if (ok) {
        fence_proxy_async_global();
        mbar_arrive_expect_tx(r_full, 32768);
        bulk_g2s_hint(sm + ST_R, rec(0) + kROff, 32768, r_full, pol_once);
        mbar_arrive_expect_tx(o_full, 32768);
        bulk_g2s_hint(sm + ST_O, rec(0) + kOOff, 32768, o_full, pol_once);
        r_in = o_in = 0;
      } else {
        *abort_flag = 1;
      }
    }
    ok = named_sync_and(2, 128, ok);
    for (int j = 0; j < nb && ok; ++j) {
      const uint32_t par = (uint32_t)j & 1u;
      const uint32_t tbuf = ST_TO + 128u * (uint32_t)(j & 1);
      bool mine = true;
      if (lead) {
        // R_j S_j behind M_j S_j, then O''_j I; TMEM buffer j & 1 was read two blocks ago
        mine = wait_or_abort(ms_issued, par, abort_flag, tmo) && wait_or_abort(r_full, par, abort_flag, tmo);
        if (mine) {
          r_in = -1;
          fence_after_sync();
#pragma unroll
          for (int k16 = 0; k16 < 8; ++k16)
            mma_ss(tmem_at(tm, 0, tbuf), dR + mstep(k16), dS + mstep(k16), id_mn, k16 > 0);
          mma_commit(rs_done);
          issued = true;
        }
        mine = mine && wait_or_abort(o_full, par, abort_flag, tmo);
        if (mine) {
          o_in = -1;
          fence_after_sync();
#pragma unroll
          for (int k16 = 0; k16 < 8; ++k16)
            mma_ss(tmem_at(tm, 0, tbuf), dO + mstep(k16), dI + mstep(k16), id_mn, 1);
          mma_commit(od_done);
        }
        if (mine && j + 1 < nb) {
          mine = acquire_through(flags, j + 1, nb, ready, a.token, a.status, tmo);
          // R_j, then O''_j, consumed as their products complete: the next block's parts
          mine = mine && wait_or_abort(rs_done, par, abort_flag, tmo);
          if (mine) {
            fence_proxy_async_global();
            mbar_arrive_expect_tx(r_full, 32768);
            bulk_g2s_hint(sm + ST_R, rec(j + 1) + kROff, 32768, r_full, pol_once);
            r_in = j + 1;
          }
          mine = mine && wait_or_abort(od_done, par, abort_flag, tmo);
          if (mine) {
            mbar_arrive_expect_tx(o_full, 32768);
            bulk_g2s_hint(sm + ST_O, rec(j + 1) + kOOff, 32768, o_full, pol_once);
            o_in = j + 1;
          }
        }
        if (!mine) *abort_flag = 1;
        bulk_wait_read();   // the previous block's TMA store has read the staging tile
      }
      mine = mine && wait_or_abort(od_done, par, abort_flag, tmo);
      uint4 po[16];   // token row r of O_j in bf16, 8 channels per entry
      if (mine) {
        fence_after_sync();
#pragma unroll
        for (int n0 = 0; n0 < D; n0 += 64) {
          float ov[64];
          tmem_ld32(tmem_at(tm, lane_base, tbuf + n0), *reinterpret_cast<float(*)[32]>(ov));
          tmem_ld32(tmem_at(tm, lane_base, tbuf + n0 + 32), *reinterpret_cast<float(*)[32]>(ov + 32));
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              __nv_bfloat162 hh = __floats2bfloat162_rn(ov[8 * i + 2 * e], ov[8 * i + 2 * e + 1]);
              w[e] = *reinterpret_cast<uint32_t*>(&hh);
            }
            po[(n0 >> 3) + i] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
      fence_before_sync();
      mine = named_sync_and(2, 128, mine);   // staging tile free (lead waited above); TMEM buffer read
      if (mine) {
#pragma unroll
        for (int i = 0; i < 16; ++i)
          *reinterpret_cast<uint4*>(sm + ST_STG + (i >> 3) * 16384 + swz_off(r, 8 * (i & 7))) = po[i];
      }
      fence_proxy_async();   // staged rows, read next by the TMA store
      ok = named_sync_and(2, 128, mine);
      if (ok && lead) {
        // rows past the sequence end are not stored (TMA clips them)
#pragma unroll
        for (int pnl = 0; pnl < 2; ++pnl)
#pragma unroll
          for (int hf = 0; hf < 2; ++hf)
            tma_store_4d(o_map, sm + ST_STG + pnl * 16384 + hf * 8192, 64 * pnl, h, j * BLK + 64 * hf, b);
        bulk_commit();
      }
    }
    if (lead) {
      if (issued) {
        mma_commit(&fin[1]);
        mbar_wait(&fin[1], 0u, 100000000ull);
      }
      if (r_in >= 0) mbar_wait(r_full, (uint32_t)r_in & 1u, 100000000ull);
      if (o_in >= 0) mbar_wait(o_full, (uint32_t)o_in & 1u, 100000000ull);
      bulk_wait_all();
    }
  }
  if (tid == 0 && *abort_flag) set_status(a.status, KDA_ERR_TIMEOUT);
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  if (warp == 0) tmem_dealloc(tm, 512);
}

template <typename TIn>
__global__ void __launch_bounds__(256, 1) kda_tc_prep(PrepArgs a, const __grid_constant__ PrepMaps mp) {
  extern __shared__ uint8_t dyn[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dyn) + 1023) & ~uintptr_t(1023));
  uint8_t* KK = sm + OFF_KK;
  uint8_t* QQ = sm + OFF_QQ;
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
  float* tot = egl + 128;                                   // [8 octets][128]: log decay over each octet
  float* gscr = tot + 8 * 128;                              // [8 octets][64]: Gram pairs inside each octet
  uint64_t* bar = reinterpret_cast<uint64_t*>(gscr + 8 * 64);   // [0] MMA, [1] v tile, [2] log alpha, k, q
  uint64_t* v_bar = bar + 1;
  uint64_t* in_bar = bar + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 4);
  uint64_t* bar2 = bar + 5;                                      // second MMA group of a round

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int sub = warp & 3, chalf = warp >> 2;

  if (*(volatile uint32_t*)a.status == KDA_ERR_TIMEOUT) return;   // an earlier CTA gave up: skip the work
  if ((int)blockIdx.x < a.n_state) {
    state_role(a, &mp.o, sm);
    return;
  }
  // record CTA pcta of npcta: units pcta, pcta + npcta, ...
  const int pcta = (int)blockIdx.x - a.n_state, npcta = (int)gridDim.x - a.n_state;
  // inputs are read once; records stay in L2 for the state CTAs of the same launch
  const uint64_t pol_in = l2_policy_evict_first();
  const uint64_t pol_rec = a.n_state > 0 ? l2_policy_evict_last() : l2_policy_evict_first();
  if (warp == 0) { tmem_alloc(tmem_slot, 512); tmem_relinquish(); }
  if (tid == 0) {
    mbar_init(bar, 1);
    mbar_init(v_bar, 1);
    mbar_init(in_bar, 1);
    mbar_init(bar2, 1);
    fence_mbar_init();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tm = *tmem_slot;
  uint32_t phase = 0, phase2 = 0, v_phase = 0, in_phase = 0;
  bool alive = true;
  bool in_inflight = false, v_inflight = false;   // thread 0: TMA loads not yet waited for
  // batch item, head and first token of the sub-chunk this CTA processes after (u, s_)
  auto next_sub = [&](int u, int s_, int& nb_, int& nh_, int& nt0_) -> bool {
    const int nu = s_ == 0 ? u : u + npcta;
    if (nu >= a.n_units) return false;
    const int blk_ = nu / a.BH, bh_ = nu - blk_ * a.BH;
    nb_ = bh_ / a.H;
    nh_ = bh_ - nb_ * a.H;
    nt0_ = blk_ * BLK + (s_ ^ 1) * SUB;
    return true;
  };
  // beta as raw bf16 bits: loaded unconditionally from a clamped index and masked where it is
  // used, one sub-chunk later, so nothing waits for the load meanwhile
  auto load_beta = [&](int b_, int h_, int t_) -> uint32_t {
    const int64_t tc = t_ < a.N ? t_ : a.N - 1;
    return (uint32_t)static_cast<const uint16_t*>(a.beta)[((int64_t)b_ * a.N + tc) * a.H + h_];
  };
  uint32_t beta_next = 0u;
  bool beta_ok = false;
  if (tid < SUB && pcta < a.n_units) {
    const int bh_ = pcta % a.BH;   // unit pcta: block pcta / BH, sub-chunk 0
    const int t_ = (pcta / a.BH) * BLK + tid;
    beta_next = load_beta(bh_ / a.H, bh_ % a.H, t_);
    beta_ok = t_ < a.N;
  }
  // v of the sub-chunk starting at token t0_ -> VV (thread 0)
  auto issue_v = [&](int b_, int h_, int t0_) {
    mbar_arrive_expect_tx(v_bar, 2 * 8192);
#pragma unroll
    for (int pnl = 0; pnl < 2; ++pnl) tma_load_4d_hint(VV + pnl * 8192, &mp.v, 64 * pnl, h_, t0_, b_, v_bar, pol_in);
  };
  bool v_early = false;   // thread 0: the sub-chunk's v is already on its way
  // log alpha, k and q of sub-chunk s_ of unit u -> G (thread 0)
  auto issue_in = [&](int u, int s_) {
    const int blk_ = u / a.BH, bh_ = u - blk_ * a.BH;
    const int b_ = bh_ / a.H, h_ = bh_ - b_ * a.H, t0_ = blk_ * BLK + s_ * SUB;
    mbar_arrive_expect_tx(in_bar, 32768 + 4 * 8192);
    tma_load_4d_hint(G, &mp.la, 0, h_, t0_, b_, in_bar, pol_in);
#pragma unroll
    for (int pnl = 0; pnl < 2; ++pnl) {
      tma_load_4d_hint(G + G_IN + pnl * 16384, &mp.k, 64 * pnl, h_, t0_, b_, in_bar, pol_in);
      tma_load_4d_hint(G + G_IN + pnl * 16384 + 8192, &mp.q, 64 * pnl, h_, t0_, b_, in_bar, pol_in);
    }
  };
  // self-test of the bounded waits: the first record CTA never issues its first inputs, so its wait gives up
  if (tid == 0 && pcta < a.n_units && !(a.fault == 1 && pcta == 0)) {
    issue_in(pcta, 0);
    in_inflight = true;
  }

  // operand descriptors of the fixed tiles (stepped along K by kstep / mstep)
  const uint64_t dM2k = kdesc0(smem_u32(QQ));                             // M_2: [128][128], panels 16 KB
  const uint64_t dKKm = mdesc0(smem_u32(KK), 8192), dQQm = mdesc0(smem_u32(QQ), 8192);   // K Gamma, Q Gamma
  const uint64_t dWUk = kdesc0(smem_u32(KK));                             // [W^T; U~^T]: [256][64]
  const uint64_t dKNm = mdesc0(smem_u32(KN), 8192);
  const uint64_t dVVm = mdesc0(smem_u32(VV), 8192);
  const uint64_t dTTk = kdesc0(smem_u32(TT)), dPPk = kdesc0(smem_u32(PP));
  const uint64_t dM1m = mdesc0(smem_u32(M1), 16384), dB1m = mdesc0(smem_u32(B1), 16384);
  const uint64_t dGrow = kdesc0(smem_u32(G + G_ROW)), dGcol = kdesc0(smem_u32(G + G_COL));
  const uint64_t dGdcol = kdesc0(smem_u32(G + G_DCOL));
  const uint64_t dQ2m = mdesc0(smem_u32(KK), 16384);                      // Q^_2^T: [128 channels][64 tokens]
  const uint64_t dUk = kdesc0(smem_u32(VV));                              // U~^T
  const uint32_t id_gram = idesc_f16(64, 32, false, false);
  const uint32_t id_direct = idesc_f16(128, 64, false, false);
  const uint32_t id_128x64_kk = idesc_f16(128, 64, false, false);
  const uint32_t id_128x64_kk_neg = idesc_f16(128, 64, false, false, true);   // D (+)= -A B
  const uint32_t id_128x64_mnmn = idesc_f16(128, 64, true, true);
  const uint32_t id_128x64_mnk = idesc_f16(128, 64, true, false);
  const uint32_t id_128x256_mnk = idesc_f16(128, 256, true, false);
  const uint32_t id_128x128_kmn = idesc_f16(128, 128, false, true);

  // front-pass role of this thread: octet fo (tokens 8 fo .. 8 fo + 7), channels 4 lane .. 4 lane + 3
  const int fo = warp, fpnl = lane >> 4, fpc = (4 * lane) & 63;

  // thread 0: the unit whose record stores are committed but not yet published (with state CTAs)
  int pub_pending = -1;
  auto publish = [&](int u) {
    const int blk_ = u / a.BH, bh_ = u - blk_ * a.BH;
    fence_proxy_async_global();   // the completed bulk stores, ordered before the release
    st_release_gpu(a.flags + (int64_t)bh_ * a.n_blocks + blk_, a.token);
  };

  for (int unit = pcta; unit < a.n_units && alive; unit += npcta) {
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
      // log alpha, k, q in G (issued during the previous sub-chunk, after its inverse), v in VV
      // (issued once the previous sub-chunk's products were done): TMA, rows past the sequence end
      // read as zero (log alpha too: alpha = 1)
      if (tid == 0 && alive) {
        if (!v_early) issue_v(b, h, (int)t0);
        v_early = false;
        v_inflight = true;
      }
      if (tid < SUB) {
        // beta of this sub-chunk was read one sub-chunk ago; read the next one now
        beta_s[tid] = beta_ok ? __uint_as_float(beta_next << 16) : 0.f;
        int nb_ = b, nh_ = h, nt0_ = (int)t0;
        const bool more = next_sub(unit, s, nb_, nh_, nt0_);
        beta_ok = more && nt0_ + tid < a.N;
        beta_next = load_beta(more ? nb_ : b, more ? nh_ : h, more ? nt0_ + tid : (int)t0);
      }
      {
        const bool ok_in = wait_tma(in_bar, in_phase, a.status, alive, a.wait_ns);
        if (tid == 0 && ok_in) in_inflight = false;
        alive = __syncthreads_and(ok_in);
      }
      // ---------------- front pass ----------------
      // Thread: octet fo (tokens 8 fo .. 8 fo + 7), four channels.  Per-token factors referenced
      // to the sub-chunk start, all <= 1: Gamma_t = e^{g_t} (rows of K Gamma, Q Gamma) and
      // e^{g_l - g_t} (rows of K~).  The pairwise decays e^{g_r - g_i} of A and P take one of two
      // factorisations, chosen for the whole sub-chunk:
      //   direct: e^{g_r - g_31} e^{g_31 - g_i}, one tensor-core product, when every factor and
      //     operand stays far inside fp16 (the decay over each half of the sub-chunk at most
      //     kHalfRange nats in every channel, |k|, |q| <= kMagRange);
      //   levels: split points between r and i (see the file header), for any gates.
      float al[8][4], ls[8][4], kx[8][4], qx[8][4];
      bool big = false;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int tok = 8 * fo + j;
        const float4 x = *reinterpret_cast<const float4*>(LA + tok * D + 4 * lane);
        const float xv[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          al[j][c] = __expf(xv[c]);
          ls[j][c] = (j ? ls[j - 1][c] : 0.f) + xv[c];   // log decay from the octet start
        }
        ld_act4(G + G_IN + fpnl * 16384 + swz_off(tok, fpc), kx[j], (TIn*)nullptr);
        ld_act4(G + G_IN + fpnl * 16384 + swz_off(64 + tok, fpc), qx[j], (TIn*)nullptr);
#pragma unroll
        for (int c = 0; c < 4; ++c) big |= fabsf(kx[j][c]) > kMagRange || fabsf(qx[j][c]) > kMagRange;
      }
      *reinterpret_cast<float4*>(tot + fo * D + 4 * lane) = make_float4(ls[7][0], ls[7][1], ls[7][2], ls[7][3]);
      if (tid == 0) bulk_wait_read_but1();   // the staged record store from KN has read it
      __syncthreads();                  // octet log totals published; log alpha, k, q read (G is free)
      // log decay before this octet, over each half, and the choice of factorisation
      float gb[4], h0[4], h1[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) gb[c] = h0[c] = h1[c] = 0.f;
#pragma unroll
      for (int o = 0; o < 8; ++o) {
        const float4 t4 = *reinterpret_cast<const float4*>(tot + o * D + 4 * lane);
        const float tv[4] = {t4.x, t4.y, t4.z, t4.w};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          if (o < fo) gb[c] += tv[c];
          if (o < 4) h0[c] += tv[c]; else h1[c] += tv[c];
        }
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) big |= h0[c] < -kHalfRange || h1[c] < -kHalfRange;
      const bool levels = __syncthreads_or(big);
      if (fo == 0)   // Gamma_l = e^{g_l}
        *reinterpret_cast<float4*>(egl + 4 * lane) =
            make_float4(__expf(h0[0] + h1[0]), __expf(h0[1] + h1[1]), __expf(h0[2] + h1[2]), __expf(h0[3] + h1[3]));
      if (!levels) {
        // direct: x = g_t - g_31, within +-kHalfRange; Gamma_t = e^{g_31} e^x, e^{g_l - g_t} = e^{g_l - g_31} e^{-x}.
        // e^x runs forward through the octet from its first token (times alpha), e^{-x} backward from
        // its last; channel pairs go through the packed fp32x2 multiply.
        uint64_t ep[8][2], en[8][2], e31[2], el31[2];
#pragma unroll
        for (int pc = 0; pc < 2; ++pc) {
          const int c0 = 2 * pc, c1 = 2 * pc + 1;
          e31[pc] = f2pack(__expf(h0[c0]), __expf(h0[c1]));
          el31[pc] = f2pack(__expf(h1[c0]), __expf(h1[c1]));
          ep[0][pc] = f2pack(__expf(gb[c0] + ls[0][c0] - h0[c0]), __expf(gb[c1] + ls[0][c1] - h0[c1]));
          en[7][pc] = f2pack(__expf(h0[c0] - gb[c0] - ls[7][c0]), __expf(h0[c1] - gb[c1] - ls[7][c1]));
#pragma unroll
          for (int j = 1; j < 8; ++j) ep[j][pc] = f2mul(ep[j - 1][pc], f2pack(al[j][c0], al[j][c1]));
#pragma unroll
          for (int j = 6; j >= 0; --j) en[j][pc] = f2mul(en[j + 1][pc], f2pack(al[j + 1][c0], al[j + 1][c1]));
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int tok = 8 * fo + j;
          const uint32_t o128 = swz_off(tok, fpc), oq = swz_off(64 + tok, fpc);
          uint64_t kg[2], qg[2], kt[2], rk[2], rq[2], ck[2];
#pragma unroll
          for (int pc = 0; pc < 2; ++pc) {
            const uint64_t k2 = f2pack(kx[j][2 * pc], kx[j][2 * pc + 1]);
            const uint64_t q2 = f2pack(qx[j][2 * pc], qx[j][2 * pc + 1]);
            const uint64_t gam = f2mul(e31[pc], ep[j][pc]), ktf = f2mul(el31[pc], en[j][pc]);
            kg[pc] = f2mul(k2, gam);
            qg[pc] = f2mul(q2, gam);
            kt[pc] = f2mul(k2, ktf);
            rk[pc] = f2mul(k2, ep[j][pc]);
            rq[pc] = f2mul(q2, ep[j][pc]);
            ck[pc] = f2mul(k2, en[j][pc]);
          }
          st_h4x2(KK + fpnl * 8192 + o128, kg[0], kg[1]);
          st_h4x2(QQ + fpnl * 8192 + o128, qg[0], qg[1]);
          st_h4x2(KN + fpnl * 8192 + o128, kt[0], kt[1]);
          // Gram operands: rows [K e^x; Q e^x] (M = 128), columns K e^{-x} (N = 64)
          uint8_t* rt = G + G_ROW + fpnl * 16384;
          st_h4x2(rt + o128, rk[0], rk[1]);
          st_h4x2(rt + oq, rq[0], rq[1]);
          st_h4x2(G + G_DCOL + fpnl * 8192 + o128, ck[0], ck[1]);
        }
      } else {
        // levels: prefix (pre) and suffix (suf) products of the gates within the octet, and across
        // octets the octet totals
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
        float gp[4], ka[4], f5[4], f4[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) gp[c] = ka[c] = f5[c] = f4[c] = 1.f;
#pragma unroll
        for (int o = 0; o < 8; ++o) {
          const float4 t4 = *reinterpret_cast<const float4*>(tot + o * D + 4 * lane);
          const float tv[4] = {__expf(t4.x), __expf(t4.y), __expf(t4.z), __expf(t4.w)};
          const bool in5 = (fo & 4) ? (o >= 4 && o < fo) : (o > fo && o < 4);
          const bool in4 = (fo & 2) ? ((fo & 1) && o == fo - 1) : (!(fo & 1) && o == fo + 1);
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            if (o < fo) gp[c] *= tv[c];
            if (o > fo) ka[c] *= tv[c];
            if (in5) f5[c] *= tv[c];
            if (in4) f4[c] *= tv[c];
          }
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int tok = 8 * fo + j;
          float g[4], kt[4], r3[4], r4[4], r5[4];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            g[c] = gp[c] * pre[j][c];
            kt[c] = suf[j][c] * ka[c];
            r3[c] = (fo & 1) ? pre[j][c] : suf[j][c];
            r4[c] = (fo & 2) ? f4[c] * pre[j][c] : suf[j][c] * f4[c];
            r5[c] = (fo & 4) ? f5[c] * pre[j][c] : suf[j][c] * f5[c];
          }
          const float* kk = kx[j];
          const float* qq = qx[j];
          const uint32_t o128 = swz_off(tok, fpc);
          st_h4(KK + fpnl * 8192 + o128, kk[0] * g[0], kk[1] * g[1], kk[2] * g[2], kk[3] * g[3]);
          st_h4(QQ + fpnl * 8192 + o128, qq[0] * g[0], qq[1] * g[1], qq[2] * g[2], qq[3] * g[3]);
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
      // ---------------- Gram on the tensor cores ----------------
      // direct: [K e^x; Q e^x] (K e^{-x})^T, one M = 128 product: A in rows 0-63, P in rows 64-127.
      // levels: level l pairs the 32 tokens with bit l set (rows: k and q, scaled by the decay
      // from the level's split point) with the 32 with bit l clear (columns: k, scaled by the
      // decay up to it): entry (r, i) is valid when r and i share their bits above l, and then
      // equals sum_c k_r (or q_r) k_i e^{g_r - g_i}.  Levels 5, 4, 3 cover every pair in different
      // octets; pairs inside an octet follow on the CUDA cores.
      if (tid == 0 && alive) {
        fence_after_sync();
        if (!levels) {
#pragma unroll
          for (int k16 = 0; k16 < 8; ++k16)
            mma_ss(tmem_at(tm, 0, C_G), dGrow + kstep(k16, 16384), dGdcol + kstep(k16, 8192), id_direct, k16 > 0);
        } else {
#pragma unroll
          for (int li = 0; li < 3; ++li)
#pragma unroll
            for (int k16 = 0; k16 < 8; ++k16)
              mma_ss(tmem_at(tm, 0, C_G + 32 * li), dGrow + ((uint32_t)li * 16384 >> 4) + kstep(k16, 8192),
                     dGcol + ((uint32_t)li * 8192 >> 4) + kstep(k16, 4096), id_gram, k16 > 0);
        }
        mma_commit(bar);
      }
      if (levels) {
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
      if (tid == 0) bulk_wait_read();   // every staged record store has read TT and PP
      alive = __syncthreads_and(wait_mma(bar, phase, a.status, alive, a.wait_ns));
      fence_after_sync();
      if (!levels) {
        // A rows (TMEM lanes 0-63) -> As (beta, strict lower); P rows (lanes 64-127) -> PP (lower)
        const int row = 32 * sub + lane;
        const int col0 = 32 * chalf;
        float v[32];
        tmem_ld32(tmem_at(tm, 32 * sub, C_G + col0), v);
        tmem_wait_ld();
        if (sub < 2) {
          const float bt = beta_s[row];
#pragma unroll
          for (int j = 0; j < 32; j += 4)
            *reinterpret_cast<float4*>(As + row * LDA + col0 + j) =
                make_float4(col0 + j < row ? bt * v[j] : 0.f, col0 + j + 1 < row ? bt * v[j + 1] : 0.f,
                            col0 + j + 2 < row ? bt * v[j + 2] : 0.f, col0 + j + 3 < row ? bt * v[j + 3] : 0.f);
        } else {
          const int r = row - 64;
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = (col0 + j <= r) ? v[j] : 0.f;
          st_row32_h(PP, r, col0, v);
        }
      } else {
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
      {
        // v of this sub-chunk (issued a sub-chunk ago); a caller's bf16 v becomes the fp16 operand in place
        const bool ok_v = wait_tma(v_bar, v_phase, a.status, alive, a.wait_ns);
        if (tid == 0 && ok_v) v_inflight = false;
        if constexpr (!kIsHalf<TIn>) {
          for (int e = tid; e < 1024; e += 256) {
            const int r = e >> 4, ch = (e & 15) * 8;
            uint4* p = reinterpret_cast<uint4*>(VV + (ch >> 6) * 8192 + swz_off(r, ch & 63));
            const uint4 u = *p;
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
            float f[8];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float2 t2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
              f[2 * i] = t2.x;
              f[2 * i + 1] = t2.y;
            }
            *p = pack8(f);
          }
        }
        fence_proxy_async();
        fence_before_sync();
        alive = __syncthreads_and(ok_v);
      }
      // T = (I + A)^{-1} Diag(beta) -> TT; then W^T = (K Gamma)^T T^T and U~^T = V^T T^T (M = 128
      // channels, N = 64 tokens)
      inverse64(As, Xs, Ys, TT, beta_s);
      fence_before_sync();
      __syncthreads();   // T published
      // two issuing threads in different warps: thread 0 the W^T products (commit on bar), thread 32
      // the U~^T products (commit on bar2)
      if ((tid == 0 || tid == 32) && alive) {
        fence_after_sync();
        const uint32_t dmine = tid == 0 ? C_W : C_U;
        const uint64_t amine = tid == 0 ? dKKm : dVVm;
#pragma unroll
        for (int k16 = 0; k16 < 4; ++k16)
          mma_ss(tmem_at(tm, 0, dmine), amine + mstep(k16), dTTk + kstep(k16, 8192), id_128x64_mnk, k16 > 0);
        mma_commit(tid == 0 ? bar : bar2);
      }
      if (tid == 0 && alive) {
        // A, X, Y consumed: G takes the log alpha, k and q of this CTA's next sub-chunk
        const int nunit = s == 0 ? unit : unit + npcta;
        if (nunit < a.n_units) {
          issue_in(nunit, s ^ 1);
          in_inflight = true;
        }
        // the previous unit's record, stored at its end, is published while the products run (the
        // proxy fence may wait for this thread's copies in flight; the products take longer)
        if (pub_pending >= 0) {
          bulk_wait_all();
          publish(pub_pending);
          pub_pending = -1;
        }
      }
      {
        const bool w1 = wait_mma(bar, phase, a.status, alive, a.wait_ns);
        alive = __syncthreads_and(wait_mma(bar2, phase2, a.status, w1, a.wait_ns));
      }
      fence_after_sync();
      // W^T -> KK, U~^T -> VV: [128 channels][64 tokens] fp16, K-major B operands of the next round
      {
        const int c = 32 * sub + lane, t0c = 32 * chalf;
        float w[32], u[32];
        tmem_ld32(tmem_at(tm, 32 * sub, C_W + t0c), w);
        tmem_ld32(tmem_at(tm, 32 * sub, C_U + t0c), u);
        tmem_wait_ld();
        st_row32_h(KK, c, t0c, w);
        st_row32_h(VV, c, t0c, u);
        // T consumed: TT becomes the 64x64 identity, the A operand that adds Q Gamma to -P W
        for (int e = tid; e < 512; e += 256) {
          const int ir = e >> 3, c8 = e & 7;
          float v8[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) v8[j] = (8 * c8 + j == ir) ? 1.f : 0.f;
          *reinterpret_cast<uint4*>(TT + swz_off(ir, 8 * c8)) = pack8(v8);
        }
      }
      fence_proxy_async();
      fence_before_sync();
      __syncthreads();
      // ---------------- K~^T [W | U~], then R^T = (Q Gamma)^T - W^T P^T and O'^T = U~^T P^T ----------------
      // [MK | BK] = K~^T [W | U~] is one N = 256 product over [W^T; U~^T].  R and O' are formed
      // transposed (M = 128 channels, N = 64 tokens; the identity tile adds (Q Gamma)^T), so Q Gamma
      // is consumed on the tensor core and KK, VV, QQ are free once the round completes.
      if (tid == 0 && alive) {   // first group: thread 0
        fence_after_sync();
#pragma unroll
        for (int k16 = 0; k16 < 4; ++k16)
          mma_ss(tmem_at(tm, 0, C_MK), dKNm + mstep(k16), dWUk + kstep(k16, 32768), id_128x256_mnk, k16 > 0);
        mma_commit(bar);
      }
      if (tid == 32 && alive) {  // second group: thread 32
        fence_after_sync();
#pragma unroll
        for (int k16 = 0; k16 < 4; ++k16) {
          const uint64_t pt = dPPk + kstep(k16, 8192);   // P^T: P's rows are the K-major B operand
          mma_ss(tmem_at(tm, 0, C_RT), dWUk + kstep(k16, 16384), pt, id_128x64_kk_neg, k16 > 0);
          mma_ss(tmem_at(tm, 0, C_OT), dUk + kstep(k16, 16384), pt, id_128x64_kk, k16 > 0);
        }
#pragma unroll
        for (int k16 = 0; k16 < 4; ++k16)
          mma_ss(tmem_at(tm, 0, C_RT), dQQm + mstep(k16), dTTk + kstep(k16, 8192), id_128x64_mnk, 1);
        mma_commit(bar2);
      }
      if (tid == 0) bulk_wait_read();   // staged records read: their tiles may be rewritten
      alive = __syncthreads_and(wait_mma(bar, phase, a.status, alive, a.wait_ns));
      fence_after_sync();
      const int row = 32 * sub + lane;        // M=128 layout row
      // M_s = Diag(Gamma_l) - K~^T W: M_1 -> M1 tile and B_1 -> B1 tile while the second group runs;
      // M_2 -> KK, QQ (combine A operand) once the second group no longer reads W^T and Q Gamma there
      auto m_epilogue = [&](uint8_t* dst, bool with_b) {
        for (int cb = 0; cb < 2; ++cb) {
          const int col0 = 64 * chalf + 32 * cb;
          float m[32];
          tmem_ld32(tmem_at(tm, 32 * sub, C_MK + col0), m);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) m[j] = (row == col0 + j ? egl[row] : 0.f) - m[j];
          st_row32_h(dst + chalf * 16384, row, col0 & 63, m);
          if (with_b) {
            float bv[32];
            tmem_ld32(tmem_at(tm, 32 * sub, C_BK + col0), bv);
            tmem_wait_ld();
            st_row32_h(B1 + chalf * 16384, row, col0 & 63, bv);
          }
        }
      };
      // transposed results (M = 128 layout: lane = channel) -> a swizzled [128 channels][64 tokens] panel
      auto t_epilogue = [&](uint32_t col, uint8_t* panel) {
        float v[32];
        tmem_ld32(tmem_at(tm, 32 * sub, col + 32 * chalf), v);
        tmem_wait_ld();
        st_row32_h(panel, row, 32 * chalf, v);
      };
      if (s == 0) m_epilogue(M1, true);
      alive = alive && wait_mma(bar2, phase2, a.status, alive, a.wait_ns);
      fence_after_sync();
      if (tid == 0 && alive) {
        // U~^T (VV) consumed: the next sub-chunk's v may land now
        int nb_, nh_, nt0_;
        if (next_sub(unit, s, nb_, nh_, nt0_)) {
          issue_v(nb_, nh_, nt0_);
          v_early = true;
          v_inflight = true;
        }
      }
      if (s == 0) {
        // R_1^T and O'_1^T, staged for the record (token panel / half 0): TT and PP, KN
        t_epilogue(C_RT, TT);
        t_epilogue(C_OT, KN);
        fence_proxy_async();
        fence_before_sync();
        alive = __syncthreads_and(alive);
        if (tid == 0) {
          bulk_s2g_hint(gO, KN, 16384, pol_rec);   // KN first, as its own group: the next sub-chunk rewrites it first
          bulk_commit();
          bulk_s2g_hint(gR, TT, 16384, pol_rec);
          bulk_commit();
        }
      } else {
        m_epilogue(QQ, false);
        // Q^_2^T -> KK (MN-major B operand of the combine)
        t_epilogue(C_RT, KK);
        fence_proxy_async();
        fence_before_sync();
        alive = __syncthreads_and(alive);
        // ---------------- combine ----------------
        if ((tid == 0 || tid == 32) && alive) {   // thread 0: M, B (bar); thread 32: R_2^T, O''_2^T (bar2)
          fence_after_sync();
          if (tid == 0) {
#pragma unroll
            for (int k16 = 0; k16 < 8; ++k16) {
              const uint64_t m2 = dM2k + kstep(k16, 16384);
              mma_ss(tmem_at(tm, 0, C_MK), m2, dM1m + mstep(k16), id_128x128_kmn, k16 > 0);   // M = M_2 M_1
              mma_ss(tmem_at(tm, 0, C_BK), m2, dB1m + mstep(k16), id_128x128_kmn, 1);         // B = B_2 + M_2 B_1
            }
            mma_commit(bar);
          } else {
#pragma unroll
            for (int k16 = 0; k16 < 8; ++k16) {
              // M_1, B_1 serve transposed as MN-major A operands (their images as B operands)
              const uint64_t q2 = dQ2m + mstep(k16);
              mma_ss(tmem_at(tm, 0, C_RT), dM1m + mstep(k16), q2, id_128x64_mnmn, k16 > 0);   // R_2^T = M_1^T Q^_2^T
              mma_ss(tmem_at(tm, 0, C_OT), dB1m + mstep(k16), q2, id_128x64_mnmn, 1);         // O''_2^T += B_1^T Q^_2^T
            }
            mma_commit(bar2);
          }
        }
        if (tid == 0) bulk_wait_read();   // staged records read: their tiles may be rewritten
        {
          const bool w1 = wait_mma(bar, phase, a.status, alive, a.wait_ns);
          alive = __syncthreads_and(wait_mma(bar2, phase2, a.status, w1, a.wait_ns));
        }
        fence_after_sync();
        // records staged in tiles the combine products no longer read:
        //   M -> M1 region, B -> B1 region, R_2^T -> TT/PP region, O''_2^T -> KN region
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
        t_epilogue(C_RT, TT);
        t_epilogue(C_OT, KN);
        fence_proxy_async();
        fence_before_sync();
        __syncthreads();
        if (tid == 0) {
          bulk_s2g_hint(gO + 16384, KN, 16384, pol_rec);   // KN first, as its own group
          bulk_commit();
          bulk_s2g_hint(gM, M1, 32768, pol_rec);
          bulk_s2g_hint(gB, B1, 32768, pol_rec);
          bulk_s2g_hint(gR + 16384, TT, 16384, pol_rec);
          bulk_commit();
          if (a.n_state > 0) pub_pending = unit;
        }
        fence_before_sync();
        __syncthreads();   // TMEM and shared tiles free for the next unit
        fence_after_sync();
      }
    }
  }
  if (tid == 0) {
    // loads still in flight after a timeout land before the CTA exits
    if (in_inflight) mbar_wait(in_bar, in_phase, 100000000ull);
    if (v_inflight) mbar_wait(v_bar, v_phase, 100000000ull);
    bulk_wait_all();
    if (pub_pending >= 0) publish(pub_pending);
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
  // with CW <= 32, O'' is added on the tensor core (O'' I, I the CW x CW identity, MN-major), as in
  // the state role of kda_tc_prep, so both give the same bits; with CW = 64 (no room for I) the
  // output threads add it
  static constexpr bool O_MMA = CW <= 32;
  static constexpr uint32_t OFF_I = OFF_S + 32768;
  static constexpr uint32_t OFF_BAR = OFF_I + (O_MMA ? 4096 : 0);
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
  const uint32_t idesc_r = idesc_f16(128, CW, true, true);   // R: MN-major image [channels][tokens]
  const uint64_t dS = mdesc0(smem_u32(sm + CH_OFF_S), 16384);
  const int lane_base = 32 * (warp & 3);
  bool ok = true;
  if constexpr (L::O_MMA) {
    // rows 0 .. CW-1 of the identity: the K = CW operand of O'' I
    if (tid < CW) {
#pragma unroll
      for (int i = 0; i < CW / 8; ++i) {
        float e8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) e8[e] = tid == 8 * i + e ? 1.f : 0.f;
        *reinterpret_cast<uint4*>(sm + L::OFF_I + swz_off(tid, 8 * i)) = pack8(e8);
      }
    }
    fence_proxy_async();
    __syncthreads();
  }

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
    const uint64_t dR = mdesc0(smem_u32(sm + CH_OFF_B), 16384);
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
          for (int k16 = 0; k16 < 8; ++k16) mma_ss(d, da + mstep(k16), db + mstep(k16), idesc_r, k16 > 0);
          if constexpr (L::O_MMA) {
            // O'' of this slot: [token half][CW channels][64 tokens], an MN-major A operand (K = CW)
            const uint64_t dO = mdesc0(smem_u32(sm + CH_OFF_B + (j & 1) * CH_SLOT + 32768), CW_BYTES / 2);
            const uint64_t dI = mdesc0(smem_u32(sm + L::OFF_I), 16384);
#pragma unroll
            for (int k16 = 0; k16 < CW / 16; ++k16) mma_ss(d, dO + mstep(k16), dI + mstep(k16), idesc_r, 1);
          }
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
        // O'': this token half's [CW channels][64 tokens], swizzled rows
        const uint8_t* Oo = sm + CH_OFF_B + (j & 1) * CH_SLOT + 32768 + (r >> 6) * (CW_BYTES / 2);
        const int64_t tok = (int64_t)j * BLK + r;
        __nv_bfloat16* orow = obase + tok * tok_stride;
#pragma unroll
        for (int c0 = 0; c0 < CW; c0 += CK) {
          float v[CK];
          tmem_ld_n(tmem_at(tm, lane_base, CT_O + CW * (j & 1) + c0), v);
          if constexpr (!L::O_MMA) {   // O'' added here (with CW <= 32 it is in the accumulator)
            __half ou[CK];
#pragma unroll
            for (int e = 0; e < CK; ++e) ou[e] = *reinterpret_cast<const __half*>(Oo + swz_off(c0 + e, r & 63));
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < CK; ++e) v[e] += __half2float(ou[e]);
          } else {
            tmem_wait_ld();
          }
          if (tok < a.N) {
#pragma unroll
            for (int i = 0; i < CK / 8; ++i) {
              uint32_t w[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                __nv_bfloat162 hh = __floats2bfloat162_rn(v[8 * i + 2 * e], v[8 * i + 2 * e + 1]);
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
  PrepArgs pa{q, k, v, la, beta, ws, d.N, d.H, BH, n_blocks, n_units, status, wait_ns, fault,
              0, nullptr, 0u, S0, SN, static_cast<__nv_bfloat16*>(o)};
  PrepMaps mp;
  const CUtensorMapDataType adt = kIsHalf<TIn> ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if (!encode_act_map(&mp.q, q, adt, 2, d, 64, true) || !encode_act_map(&mp.k, k, adt, 2, d, 64, true) ||
      !encode_act_map(&mp.v, v, adt, 2, d, 64, true) ||
      !encode_act_map(&mp.la, la, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, d, 128, false))
    return cudaErrorInvalidValue;
  // One launch: with few (batch item, head) pairs, one CTA per pair runs the serial state pass
  // beside the record CTAs, consuming each record as soon as it is published.  Those CTAs wait on
  // the others, so the launch is cooperative (every CTA resident at once) or not made this way.
  // Each state CTA takes an SM from the records; past about a fifth of the SMs the separate
  // state-pass kernel after the record kernel costs less.
  if (!d.reuse_records && 5 * BH <= n_sm) {
    int per_sm = 0;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kda_tc_prep<TIn>, 256, PREP_SMEM)) != cudaSuccess)
      return e;
    const int grid = BH + min(n_units, n_sm - BH);
    if (per_sm >= 1 && grid <= per_sm * n_sm) {
      if (!encode_act_map(&mp.o, o, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d, 64, true)) return cudaErrorInvalidValue;
      pa.n_state = BH;
      pa.flags = reinterpret_cast<uint32_t*>(ws + (size_t)n_units * kBlockBytes);
      pa.token = 1u;
      // cleared on the stream first, so no earlier content of the workspace reads as published
      if ((e = cudaMemsetAsync(pa.flags, 0, (size_t)n_units * sizeof(uint32_t), s)) != cudaSuccess) return e;
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3((unsigned)grid);
      cfg.blockDim = dim3(256);
      cfg.dynamicSmemBytes = PREP_SMEM;
      cfg.stream = s;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeCooperative;
      attr[0].val.cooperative = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      e = cudaLaunchKernelEx(&cfg, kda_tc_prep<TIn>, pa, mp);
      if (e == cudaSuccess) {
        if (launches) *launches += 1;
        return cudaSuccess;
      }
      // a device that cannot hold the whole grid at once (a partitioned GPU, say) refuses the
      // cooperative launch: the record and state-pass kernels below do the same work
      if (e != cudaErrorCooperativeLaunchTooLarge) return e;
      (void)cudaGetLastError();
      pa.n_state = 0;
      pa.flags = nullptr;
    }
  }
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
  const size_t units = (size_t)d.B * d.H * n_blocks;
  // the records, then one publication flag per record
  return units * kBlockBytes + ((units * sizeof(uint32_t) + 255) & ~size_t(255));
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
