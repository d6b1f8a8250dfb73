// fp64-accurate matrix products on the 5th-generation int8 tensor cores: the sweep's lazy
// trailing update, and the large products of the recursive factorisation.
//
// Source of the operation: "第5章 GPTQ 实战" §5.1.8 key point 3 (lazy batch update): after a
// block of columns is quantized, its normalised errors update every later column at once,
// W[:, later] -= Err[:, block] U[block, later].  The sweep needs this product to fp64-level
// accuracy (its rounding decisions are chained), which the fp64 units give at ~37 TFLOP/s.
// Here it is formed from exact integer products instead (a splitting of the operands into
// small integer slices, as in Ozaki's scheme for accurate matrix products):
//
//   every row r of A = Err[:, block] is written A[r, k] ~ sum_{p<5} SA_p[r, k] 2^(ea_r - 7(p+1))
//   every column n of B = U[block, later] is B[k, n] ~ sum_{q<5} SB_q[n, k] 2^(eb_n - 7(q+1))
//   with SA_p, SB_q integers in [-127, 127] taken by repeated scaling by 2^7 and rounding to
//   nearest (an unbiased remainder: truncation's bias accumulated over the sweep's blocks and
//   flipped near-tie codes), and 2^ea_r > max |A[r, :]|, 2^eb_n > max |B[:, n]|.  Then
//   (A B)[r, n] ~ 2^(ea_r + eb_n) sum_{s<5} 2^(-7(s+2)) sum_{p+q=s} (SA_p SB_q^T)[r, n],
//   keeping the 15 slice pairs with p + q <= 4 (35 bits of each operand; four slices, 28
//   bits, left a few more near-tie flips than fp64 in the parity tests).  Each SA_p SB_q^T
//   is an exact int32 product (127^2 * K * 5 < 2^31 for K <= 16384).
//
// The factorisation ("第5章 GPTQ 实战" §5.1.8 key point 1, the inverse-Cholesky factor U)
// uses the same scheme with seven slices per operand (49 bits; the 28 pairs p + q <= 6,
// 7 * 127^2 * K < 2^31 for K <= 16384): its Schur complements cancel, so it keeps more bits
// than the sweep needs.
//
// Kernels: split_rows_kernel / split_cols_kernel write the slices K-major (k contiguous)
// for TMA; i8_gemm_kernel<NS, BN, NBUF, CR> runs tcgen05.mma kind::i8 (s8 x s8 -> s32) with
// the column operand's slices as the M side (128 columns of C) and the row operand's as the
// N side (BN rows of C), NS TMEM accumulators (one per s = p + q), NBUF accumulator
// buffers, a 2-stage TMA ring of all slices of a 64-wide K step (64-byte swizzle).
//  * sweep: 5 slices, 48 rows, double buffered: 111 KB of shared memory and 160 registers
//    a thread leave room on the SM for one CTA of the sweep's panel kernel, which runs
//    beside it.
//  * factor: 7 slices, 64 rows, one buffer (448 TMEM columns; 172 KB of shared memory);
//    a tile may skip the K steps where a triangular operand is zero, and a symmetric
//    update may skip the tiles strictly below the diagonal.
// In the epilogue a thread owns one column and a warp updates 32 consecutive columns of a
// row at a time (coalesced fp64 read-modify-write, loads issued together); each element of
// C is updated by exactly one thread of one CTA per launch (deterministic).
#include <cuda.h>

#include <algorithm>

#include "common.cuh"
#include "sm100.cuh"

namespace gptq {
namespace {

using namespace sm100;

constexpr int KS = 5;        // slices per operand of the sweep's update
constexpr int KSF = 7;       // slices per operand of the factorisation's products
constexpr int SBETA = 7;     // bits per slice
constexpr int IBM = 128;     // columns of C per tile (UMMA M: the column operand's slices)
constexpr int IBK = 64;      // K (bytes = int8 elements) per stage: one 64-byte swizzle row
constexpr int ISTAGES = 2;
constexpr int ITHREADS = 320;
constexpr uint32_t IWAIT = 1u << 24;

// Tile shape of one kernel instance: NS slices, BN rows of C per tile (UMMA N), NBUF TMEM
// accumulator buffers, CR rows per epilogue chunk.
template <int NS, int BN, int NBUF>
struct I8Shape {
  static constexpr int A_BYTES = NS * IBM * IBK;  // column operand slices (UMMA A)
  static constexpr int B_BYTES = NS * BN * IBK;   // row operand slices (UMMA B)
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int SMEM = ISTAGES * STAGE + 1024 + 256;
  static_assert(NBUF * NS * BN <= 512, "accumulators exceed the tensor memory");
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "UMMA N");
};
using SweepShape = I8Shape<KS, 48, 2>;
using FactorShape = I8Shape<KSF, 64, 1>;

__device__ int g_i8_status = 0;

// 2^e as a double: built from the exponent bits in the normal range, else by ldexp.
__device__ __forceinline__ double pow2(int e) {
  if (e >= -1022 && e <= 1023) return __longlong_as_double(static_cast<long long>(e + 1023) << 52);
  return ldexp(1.0, e);
}

__device__ __forceinline__ void prefetch_l2(const void* p) { asm volatile("prefetch.global.L2 [%0];" ::"l"(p)); }

// ------------------------------------------------------------------ splitting
// The NS slices of v (|v| < 1), each rounded to nearest and clamped to [-127, 127]; the
// remainder carries to the next slice.
template <int NS>
__device__ __forceinline__ void slices_of(double v, int8_t (&sl)[NS]) {
#pragma unroll
  for (int p = 0; p < NS; ++p) {
    v *= 128.0;
    const double r = fmin(fmax(rint(v), -127.0), 127.0);  // nearest, |v - r| <= 1
    v -= r;
    sl[p] = static_cast<int8_t>(r);
  }
}

// One warp per row of A (K = the row's length): the row exponent (2^e > max |row|), then NS
// slices of every element.  S is [NS][R][KP] (k contiguous, zero padded to KP).  A lane takes
// 4 consecutive k and stores 4 slice bytes at once.
template <int NS>
__global__ void split_rows_kernel(const double* __restrict__ X, int64_t ldx, int64_t R, int64_t K, int64_t KP,
                                  int8_t* __restrict__ S, int* __restrict__ e) {
  const int64_t r = static_cast<int64_t>(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (r >= R) return;
  const double* x = X + r * ldx;
  double m = 0.0;
  for (int64_t k = lane; k < K; k += 32) m = fmax(m, fabs(x[k]));
  for (int off = 16; off; off >>= 1) m = fmax(m, __shfl_xor_sync(0xffffffffu, m, off));
  const int ex = m > 0.0 ? ilogb(m) + 1 : 0;  // 2^ex > m
  if (lane == 0) e[r] = ex;
  for (int64_t k0 = 4 * lane; k0 < KP; k0 += 128) {  // KP is a multiple of 64
    uint32_t w[NS];
#pragma unroll
    for (int p = 0; p < NS; ++p) w[p] = 0;
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const int64_t k = k0 + t;
      int8_t sl[NS];
      slices_of<NS>(k < K ? ldexp(x[k], -ex) : 0.0, sl);
#pragma unroll
      for (int p = 0; p < NS; ++p) w[p] |= static_cast<uint32_t>(static_cast<uint8_t>(sl[p])) << (8 * t);
    }
#pragma unroll
    for (int p = 0; p < NS; ++p) *reinterpret_cast<uint32_t*>(S + (static_cast<int64_t>(p) * R + r) * KP + k0) = w[p];
  }
}

// Columns of B (row-major, ldy), in three steps.  col_exp_init: e[n] = -2000 (no column yet
// seen).  col_exp_kernel: per 32 columns x 256 rows, the largest ilogb(|y|) + 1, merged into e
// with atomicMax (the exponent of a column's maximum is the maximum of its exponents; the
// result does not depend on the order).  An all-zero column keeps -2000, which scales its
// (zero) slices to zero in the product.  col_slices_kernel: per 32 columns x 128 k, the
// slices transposed through shared memory into S [NS][N][KP] (k contiguous, 128-byte rows).
__global__ void col_exp_init_kernel(int* __restrict__ e, int64_t N) {
  const int64_t n = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (n < N) e[n] = -2000;
}

constexpr int CE_ROWS = 256;
__global__ void __launch_bounds__(256) col_exp_kernel(const double* __restrict__ Y, int64_t ldy, int64_t K,
                                                      int64_t N, int* __restrict__ e) {
  __shared__ int mx[8][32];
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int64_t n = static_cast<int64_t>(blockIdx.x) * 32 + tx;
  const int64_t k0 = static_cast<int64_t>(blockIdx.y) * CE_ROWS;
  int best = -2000;
  if (n < N)
    for (int64_t k = k0 + ty; k < min(K, k0 + CE_ROWS); k += 8) {
      const double v = fabs(Y[k * ldy + n]);
      if (v > 0.0) best = max(best, ilogb(v) + 1);
    }
  mx[ty][tx] = best;
  __syncthreads();
  if (ty == 0 && n < N) {
    for (int i = 1; i < 8; ++i) best = max(best, mx[i][tx]);
    if (best > -2000) atomicMax(e + n, best);
  }
}

constexpr int CS_K = 128;
template <int NS, int KW>
__global__ void __launch_bounds__(256) col_slices_kernel(const double* __restrict__ Y, int64_t ldy, int64_t K,
                                                         int64_t N, int64_t KP, int64_t kbase,
                                                         int8_t* __restrict__ S, const int* __restrict__ e) {
  constexpr int PITCH = KW + 4;  // bytes per tile row (4-byte aligned, spreads the banks)
  constexpr int WPR = KW / 4;    // 32-bit words per output row
  __shared__ __align__(16) int8_t tile[NS][32][PITCH];
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int64_t n = static_cast<int64_t>(blockIdx.x) * 32 + tx;
  const int64_t k0 = kbase + static_cast<int64_t>(blockIdx.y) * KW;
  const int ex = n < N ? max(e[n], -1100) : 0;  // a zero column's slices are zero whatever ex
  for (int kk = ty; kk < KW; kk += 8) {
    const int64_t k = k0 + kk;
    int8_t sl[NS];
    slices_of<NS>((n < N && k < K) ? ldexp(Y[k * ldy + n], -ex) : 0.0, sl);
#pragma unroll
    for (int p = 0; p < NS; ++p) tile[p][tx][kk] = sl[p];
  }
  __syncthreads();
  // rows (p, column) of KW bytes, stored as 32-bit words (consecutive threads, consecutive words)
  for (int idx = threadIdx.x; idx < NS * 32 * WPR; idx += 256) {
    const int row = idx / WPR, w = idx % WPR;
    const int p = row / 32, c = row % 32;
    const int64_t nn = static_cast<int64_t>(blockIdx.x) * 32 + c;
    if (nn < N)
      *reinterpret_cast<uint32_t*>(S + (static_cast<int64_t>(p) * N + nn) * KP + k0 + 4 * w) =
          *reinterpret_cast<const uint32_t*>(&tile[p][c][4 * w]);
  }
}

// ------------------------------------------------------------------ tcgen05 kind::i8 GEMM
// 32 lanes x 16 (or 8) consecutive 32-bit columns, the wait in the same statement.
__device__ __forceinline__ void tmem_ld_32x32b(uint32_t taddr, int (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_ld_32x32b(uint32_t taddr, int (&v)[8]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7])
      : "r"(taddr)
      : "memory");
}

// Shared-memory descriptor, K-major with 64-byte swizzle: rows of 64 bytes, 8-row atoms of 512
// bytes (stride-dimension offset); the leading-dimension offset is unused (one MMA's K, 32
// bytes, lies inside a swizzle row).
__device__ __forceinline__ uint64_t desc_sw64(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(1u) << 16;
  d |= static_cast<uint64_t>((512u >> 4) & 0x3FFFu) << 32;
  d |= 1ull << 46;
  d |= 4ull << 61;
  return d;
}

__device__ __forceinline__ void umma_i8(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Instruction descriptor of kind::i8: D s32 (2), A and B signed 8-bit (1), both K-major.
__host__ __device__ constexpr uint32_t i8_idesc(int M, int N) {
  return (2u << 4) | (1u << 7) | (1u << 10) | ((static_cast<uint32_t>(N) >> 3) << 17) |
         ((static_cast<uint32_t>(M) >> 4) << 24);
}

// K ranges of a tile (in steps of IBK) when one operand is triangular; the skipped steps
// multiply exact zeros.
enum KRange : int {
  kFullK = 0,     // every step
  kFromCol = 1,   // column operand zero for k < column (B[k, c] = U[c, k], U upper)
  kToCol = 2,     // column operand zero for k > column (B[k, c] = U[k, c], U upper)
  kFromRow = 3,   // row operand zero for k < row (A[r, k] = U[r, k], U upper)
};

struct I8Args {
  int M, N, KP;               // rows, columns, padded K
  int a_rows, b_cols;         // slice strides (rows of SA per slice, columns of SB per slice)
  const int* ea;              // [a_rows] row exponents
  const int* eb;              // [b_cols] column exponents (for columns col0 ...)
  int col0;                   // first column of this launch within SB / eb
  double* C;                  // C[r, c] for c in [0, N): C + r * ldc + c
  int64_t ldc;
  int mt, nt;
  int krange;                 // KRange
  int upper;                  // skip tiles strictly below the diagonal (square C, col0 == 0)
};

template <int BN>
struct TileOf {
  int c0, r0, kb, ke;  // first column and row, K step range [kb, ke)
  bool skip;
};

template <int BN>
__device__ __forceinline__ TileOf<BN> tile_of(const I8Args& a, int u) {
  TileOf<BN> t;
  t.c0 = (u / a.mt) * IBM;
  t.r0 = (u % a.mt) * BN;
  const int nk = a.KP / IBK;
  t.kb = 0;
  t.ke = nk;
  if (a.krange == kFromCol) t.kb = t.c0 / IBK;
  if (a.krange == kToCol) t.ke = min(nk, (t.c0 + IBM + IBK - 1) / IBK);
  if (a.krange == kFromRow) t.kb = t.r0 / IBK;
  t.kb = min(t.kb, nk - 1);  // at least one step (of zeros at worst) initialises the accumulators
  t.skip = a.upper && t.c0 + IBM <= t.r0;
  return t;
}

template <int NS, int BN, int NBUF, int CR>
__global__ void __maxnreg__(160)
    i8_gemm_kernel(const __grid_constant__ CUtensorMap ta, const __grid_constant__ CUtensorMap tb, I8Args a) {
  using Sh = I8Shape<NS, BN, NBUF>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + ISTAGES * Sh::STAGE);
  uint64_t* empty = full + ISTAGES;
  uint64_t* accf = empty + ISTAGES;
  uint64_t* acce = accf + 2;
  uint64_t* done = acce + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = static_cast<int>(gridDim.x);
  const int units = a.mt * a.nt;

  if (threadIdx.x == 0) {
    for (int s = 0; s < ISTAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accf[b], 1);
      mbar_init(&acce[b], 8);
    }
    mbar_init(done, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer: all NS slices of A and B for one 64-wide K step
      tma_prefetch_desc(&ta);
      tma_prefetch_desc(&tb);
      int stage = 0, issued = 0;
      uint32_t ph = 0;
      for (int u = blockIdx.x; u < units && ok; u += G) {
        const TileOf<BN> t = tile_of<BN>(a, u);
        if (t.skip) continue;
        for (int ks = t.kb; ks < t.ke; ++ks) {
          if (!mbar_wait(&empty[stage], ph ^ 1u, IWAIT)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + stage * Sh::STAGE;
          uint8_t* sb = sa + Sh::A_BYTES;
          mbar_arrive_expect_tx(&full[stage], Sh::STAGE);
#pragma unroll
          for (int p = 0; p < NS; ++p) {
            tma_load_2d(sa + p * IBM * IBK, &tb, &full[stage], ks * IBK, p * a.b_cols + a.col0 + t.c0);
            tma_load_2d(sb + p * BN * IBK, &ta, &full[stage], ks * IBK, p * a.a_rows + t.r0);
          }
          ++issued;
          if (++stage == ISTAGES) {
            stage = 0;
            ph ^= 1u;
          }
        }
      }
      for (int k = 0; k < min(issued, ISTAGES); ++k) {
        int s = stage - 1 - k;
        uint32_t p = ph;
        while (s < 0) {
          s += ISTAGES;
          p ^= 1u;
        }
        mbar_wait(&full[s], p, IWAIT);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- UMMA issuer: the slice pairs p + q < NS per 32-wide K substep
      constexpr uint32_t idesc = i8_idesc(IBM, BN);
      int stage = 0, cg = 0;
      uint32_t ph = 0;
      for (int u = blockIdx.x; u < units && ok; u += G) {
        const TileOf<BN> t = tile_of<BN>(a, u);
        if (t.skip) continue;
        const int b = cg % NBUF;
        const uint32_t epar = static_cast<uint32_t>((cg / NBUF) & 1);
        ++cg;
        if (!mbar_wait(&acce[b], epar ^ 1u, IWAIT)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t dbase = tmem + static_cast<uint32_t>(b * NS * BN);
        for (int ks = t.kb; ks < t.ke; ++ks) {
          if (!mbar_wait(&full[stage], ph, IWAIT)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * Sh::STAGE);
          const uint32_t sb = sa + Sh::A_BYTES;
#pragma unroll
          for (int k = 0; k < IBK / 32; ++k) {
#pragma unroll
            for (int p = 0; p < NS; ++p)
#pragma unroll
              for (int q = 0; q < NS - p; ++q) {
                const uint64_t ad = desc_sw64(sa + p * IBM * IBK + k * 32);
                const uint64_t bd = desc_sw64(sb + q * BN * IBK + k * 32);
                // pairs go p-major, so (0, s) is the first product into accumulator s: it
                // overwrites the accumulator's previous tile
                const bool first = ks == t.kb && k == 0 && p == 0;
                umma_i8(dbase + static_cast<uint32_t>((p + q) * BN), ad, bd, idesc, first ? 0u : 1u);
              }
          }
          umma_commit(&empty[stage]);
          if (++stage == ISTAGES) {
            stage = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&accf[b]);
      }
      umma_commit(done);
      mbar_wait(done, 0, IWAIT);
    }
  } else {
    // ---------------- epilogue: C[r, n] -= 2^(ea_r + eb_n - 14) sum_s acc_s 2^(-7 s).  A thread
    // owns one column n (its TMEM lane); the 4 warps of each lane quarter are split over the
    // tile's BN rows in chunks of CR (warps 2..5 take the even chunks, 6..9 the odd ones); for
    // each row the warp's 32 lanes update 32 consecutive columns (coalesced).  The CR loads of
    // C are issued together, before the accumulator reads, and the rows of this CTA's next tile
    // are prefetched into L2 while the current one is updated.
    const int quad = warp & 3;
    const int half = (warp - 2) >> 2;
    const int et = threadIdx.x - 64;  // 0..255 over the epilogue warps
    // L2 prefetch of the C lines (BN rows x 1 KiB) of tile u: 128-byte lines
    auto prefetch_tile = [&](int u) {
      for (; u < units; u += G) {
        const TileOf<BN> t = tile_of<BN>(a, u);
        if (t.skip) continue;
        for (int l = et; l < BN * (IBM / 16); l += 256) {
          const int r = t.r0 + l / (IBM / 16), cc = t.c0 + (l % (IBM / 16)) * 16;
          if (r < a.M && cc < a.N) prefetch_l2(a.C + static_cast<int64_t>(r) * a.ldc + cc);
        }
        return;
      }
    };
    prefetch_tile(blockIdx.x);
    int cg = 0;
    for (int u = blockIdx.x; u < units; u += G) {
      const TileOf<BN> t = tile_of<BN>(a, u);
      if (t.skip) continue;
      const int b = cg % NBUF;
      const uint32_t fpar = static_cast<uint32_t>((cg / NBUF) & 1);
      ++cg;
      if (!mbar_wait(&accf[b], fpar, IWAIT)) {
        ok = false;
        break;
      }
      tc_fence_after();
      prefetch_tile(u + G);
      const int c = t.c0 + quad * 32 + lane;  // column within this launch
      const bool cin = c < a.N;
      // The accumulators recombine exactly in 64-bit integers: hi = sum_{s<4} acc_s 2^(7(3-s))
      // (below 2^53), and for NS > 4 lo = sum_{s>=4} acc_s 2^(7(NS-1-s)).  The value
      // sum_s acc_s 2^(-7s) is 2^-21 (hi + lo 2^(-7(NS-4))), formed with one rounding.
      const int ec = cin ? a.eb[a.col0 + c] - 2 * SBETA - 3 * SBETA : 0;
      for (int chunk = half; chunk < BN / CR; chunk += 2) {
        const int r0 = t.r0 + chunk * CR;
        // the C loads first, so that their latency overlaps the accumulator reads
        double cv[CR];
#pragma unroll
        for (int j = 0; j < CR; ++j)
          cv[j] = (cin && r0 + j < a.M) ? a.C[static_cast<int64_t>(r0 + j) * a.ldc + c] : 0.0;
        int acc[NS][CR];
#pragma unroll
        for (int s = 0; s < NS; ++s)
          tmem_ld_32x32b(tmem + (static_cast<uint32_t>(quad * 32) << 16) +
                             static_cast<uint32_t>(b * NS * BN + s * BN + chunk * CR),
                         acc[s]);
#pragma unroll
        for (int j = 0; j < CR; ++j) {
          long long hi = acc[0][j];
#pragma unroll
          for (int s = 1; s < 4; ++s) hi = hi * (1ll << SBETA) + acc[s][j];
          double v = static_cast<double>(hi);
          if constexpr (NS > 4) {
            long long lo = acc[4][j];
#pragma unroll
            for (int s = 5; s < NS; ++s) lo = lo * (1ll << SBETA) + acc[s][j];
            v = fma(static_cast<double>(lo), pow2(-SBETA * (NS - 4)), v);
          }
          if (cin && r0 + j < a.M)
            a.C[static_cast<int64_t>(r0 + j) * a.ldc + c] = cv[j] - v * pow2(ec + a.ea[r0 + j]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acce[b]);  // this warp's reads of the accumulators are done
    }
  }
  if (!ok) atomicExch(&g_i8_status, kStatusTimeout);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<EncodeTiledFn>(p);
    return static_cast<EncodeTiledFn>(nullptr);
  }();
  return fn;
}

// rows x KP int8, boxes of 64 (K) x box_rows, 64-byte swizzle
int slice_map(CUtensorMap* tm, const int8_t* base, int64_t rows, int64_t KP, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return GPTQ_ERR_CUDA;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(KP), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(KP)};
  cuuint32_t box[2] = {IBK, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? GPTQ_OK : GPTQ_ERR_CUDA;
}

template <int NS>
int split_rows_any(cudaStream_t s, const double* X, int64_t ldx, int64_t R, int64_t K, int64_t KP, int8_t* S, int* e) {
  if (R <= 0) return GPTQ_OK;
  split_rows_kernel<NS><<<static_cast<unsigned>((R + 7) / 8), 256, 0, s>>>(X, ldx, R, K, KP, S, e);
  return after_launch();
}

template <int NS>
int split_cols_any(cudaStream_t s, const double* Y, int64_t ldy, int64_t K, int64_t N, int64_t KP, int8_t* S, int* e) {
  if (N <= 0) return GPTQ_OK;
  if (KP % 64 != 0) return GPTQ_ERR_UNSUPPORTED;
  const unsigned gx = static_cast<unsigned>((N + 31) / 32);
  col_exp_init_kernel<<<static_cast<unsigned>((N + 255) / 256), 256, 0, s>>>(e, N);
  GPTQ_TRY(after_launch());
  if (K > 0) {
    col_exp_kernel<<<dim3(gx, static_cast<unsigned>((K + CE_ROWS - 1) / CE_ROWS)), 256, 0, s>>>(Y, ldy, K, N, e);
    GPTQ_TRY(after_launch());
  }
  // KP is a multiple of 64: 128-wide chunks, and one 64-wide chunk for an odd remainder
  const int64_t full = KP / CS_K;
  if (full > 0) {
    col_slices_kernel<NS, CS_K><<<dim3(gx, static_cast<unsigned>(full)), 256, 0, s>>>(Y, ldy, K, N, KP, 0, S, e);
    GPTQ_TRY(after_launch());
  }
  if (KP % CS_K != 0) {
    col_slices_kernel<NS, 64><<<dim3(gx, 1), 256, 0, s>>>(Y, ldy, K, N, KP, full * CS_K, S, e);
    GPTQ_TRY(after_launch());
  }
  return GPTQ_OK;
}

template <int NS, int BN, int NBUF, int CR>
int gemm_any(cudaStream_t s, int64_t M, int64_t N, int64_t KP, const int8_t* SA, int64_t a_rows, const int* ea,
             const int8_t* SB, int64_t b_cols, const int* eb, int64_t col0, double* C, int64_t ldc, int max_ctas,
             int krange, int upper) {
  using Sh = I8Shape<NS, BN, NBUF>;
  if (M <= 0 || N <= 0) return GPTQ_OK;
  // Rows past a slice's end (a tile reaching beyond M) load the next slice's first rows, or
  // zeros past the last slice; they only reach accumulator rows (columns) >= M (N), which
  // the epilogue never writes.
  if (KP % IBK != 0 || KP > 16384 || M > a_rows || col0 + N > b_cols) return GPTQ_ERR_UNSUPPORTED;
  if (upper && (col0 != 0 || M != N)) return GPTQ_ERR_UNSUPPORTED;
  auto kern = i8_gemm_kernel<NS, BN, NBUF, CR>;
  GPTQ_TRY(ensure_smem_limit(reinterpret_cast<const void*>(kern), Sh::SMEM));
  CUtensorMap ta, tb;
  GPTQ_TRY(slice_map(&ta, SA, NS * a_rows, KP, BN));
  GPTQ_TRY(slice_map(&tb, SB, NS * b_cols, KP, IBM));
  I8Args a;
  a.M = static_cast<int>(M);
  a.N = static_cast<int>(N);
  a.KP = static_cast<int>(KP);
  a.a_rows = static_cast<int>(a_rows);
  a.b_cols = static_cast<int>(b_cols);
  a.ea = ea;
  a.eb = eb;
  a.col0 = static_cast<int>(col0);
  a.C = C;
  a.ldc = ldc;
  a.mt = static_cast<int>((M + BN - 1) / BN);    // row tiles
  a.nt = static_cast<int>((N + IBM - 1) / IBM);  // column tiles of 128
  a.krange = krange;
  a.upper = upper;
  const int cap = max_ctas > 0 ? std::min(max_ctas, num_sms()) : num_sms();
  const int grid = static_cast<int>(std::min<int64_t>(cap, static_cast<int64_t>(a.mt) * a.nt));
  kern<<<grid, ITHREADS, Sh::SMEM, s>>>(ta, tb, a);
  return after_launch();
}

}  // namespace

int i8_slices() { return KS; }
int i8f_slices() { return KSF; }
int64_t i8_padded_k(int64_t K) { return ((K + IBK - 1) / IBK) * IBK; }

int i8_split_rows(cudaStream_t s, const double* X, int64_t ldx, int64_t R, int64_t K, int64_t KP, int8_t* S, int* e) {
  return split_rows_any<KS>(s, X, ldx, R, K, KP, S, e);
}
int i8_split_cols(cudaStream_t s, const double* Y, int64_t ldy, int64_t K, int64_t N, int64_t KP, int8_t* S, int* e) {
  return split_cols_any<KS>(s, Y, ldy, K, N, KP, S, e);
}
int i8f_split_rows(cudaStream_t s, const double* X, int64_t ldx, int64_t R, int64_t K, int64_t KP, int8_t* S, int* e) {
  return split_rows_any<KSF>(s, X, ldx, R, K, KP, S, e);
}
int i8f_split_cols(cudaStream_t s, const double* Y, int64_t ldy, int64_t K, int64_t N, int64_t KP, int8_t* S,
                   int* e) {
  return split_cols_any<KSF>(s, Y, ldy, K, N, KP, S, e);
}

// C[r, c] -= (A B)[r, col0 + c] for r < M, c < N, from the slices of i8_split_rows (SA,
// a_rows rows per slice, exponents ea) and i8_split_cols (SB, b_cols columns per slice,
// exponents eb), K padded to KP.  The persistent grid has at most max_ctas CTAs (0: one per
// SM): a CTA takes most of an SM's shared memory, so a launch that runs beside other
// kernels leaves them SMs of their own.
int i8_gemm_sub(cudaStream_t s, int64_t M, int64_t N, int64_t KP, const int8_t* SA, int64_t a_rows, const int* ea,
                const int8_t* SB, int64_t b_cols, const int* eb, int64_t col0, double* C, int64_t ldc,
                int max_ctas) {
  return gemm_any<KS, 48, 2, 16>(s, M, N, KP, SA, a_rows, ea, SB, b_cols, eb, col0, C, ldc, max_ctas, kFullK, 0);
}

// The factorisation's products: C[r, c] -= (A B)[r, c] from seven-slice operands (i8f_split_*),
// with the K steps a triangular operand makes zero skipped (krange: 0 none, 1 B[k, c] = 0 for
// k < c, 2 B[k, c] = 0 for k > c, 3 A[r, k] = 0 for k < r) and, with upper, only the tiles
// that reach the diagonal or above (square C).
int i8f_gemm_sub(cudaStream_t s, int64_t M, int64_t N, int64_t KP, const int8_t* SA, int64_t a_rows, const int* ea,
                 const int8_t* SB, int64_t b_cols, const int* eb, double* C, int64_t ldc, int krange, int upper) {
  if (krange < kFullK || krange > kFromRow) return GPTQ_ERR_INVALID_ARG;
  return gemm_any<KSF, 64, 1, 8>(s, M, N, KP, SA, a_rows, ea, SB, b_cols, eb, 0, C, ldc, 0, krange, upper);
}

int i8_device_status(int clear) {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_i8_status, sizeof(int)) != cudaSuccess) return GPTQ_ERR_CUDA;
  if (clear) {
    int z = 0;
    if (cudaMemcpyToSymbol(g_i8_status, &z, sizeof(int)) != cudaSuccess) return GPTQ_ERR_CUDA;
  }
  return v;
}

}  // namespace gptq
