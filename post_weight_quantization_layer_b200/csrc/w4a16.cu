// Linear layer on GPTQ-quantized weights: Y = X * W_hat^T with 16-bit activations.
//
// Source: the inference side that the pages benchmark on the quantized checkpoints — the
// "gptq" skill card's kernel-backend section (ExLlama / Marlin / CUDA kernels run 4-bit
// weights against fp16 activations) and "第5章 GPTQ 实战" §5.2 (generation speed of the
// quantized model).  The weights come in the checkpoint form of export.cu: qweight
// [K*bits/32, N] int32 (codes along K, LSB first), qzeros [G, N*bits/32] int32 (zero points
// along N, LSB first), scales [G, N] fp16, g_idx [K] int32 (any order, so act-order
// checkpoints work), and
//     W_hat[n, k] = scales[g_idx[k], n] * (code[k, n] - zero[g_idx[k], n]).
// The product is defined as Y = X * round16(W_hat)^T: every dequantized weight is rounded
// once (nearest even) to the activations' 16-bit type, as a 16-bit tensor-core operand
// is, and products are accumulated in fp32.  scale * (code - zero) is exact in fp32 (an
// 11-bit scale times an integer below 2^8), so round16 sees the exact value.
//
// Two regimes:
// * decode (M <= 4 rows of X): HBM-bound on the packed weights.  gemv_kernel streams the
//   weights once (16-byte loads, coalesced along N), dequantizes in registers and
//   accumulates on the CUDA cores, split over K across CTAs; a second pass adds the K
//   splits in a fixed order (deterministic).
// * prefill / calibration (M > 4): the weights are dequantized once into a 16-bit [N, K]
//   matrix (dequant_kernel, HBM-bound), and gemm_tn_kernel multiplies on the 5th-generation
//   tensor cores: TMA loads of both K-major operands with 128-byte swizzle into a 4-stage
//   ring, tcgen05.mma kind::f16 into a TMEM accumulator of 128 x 256, persistent CTAs with
//   two accumulators in TMEM so that one tile's epilogue overlaps the next tile's MMAs.
// An act-order checkpoint (g_idx not in order) can be reordered once (sort_by_group_kernel,
// reorder_codes_kernel): its inputs sorted by group, with the permutation kept so that both
// regimes read X in the same order (the decode kernel while staging X, the tensor-core path
// through one gather).
#include <cuda.h>

#include <algorithm>

#include "common.cuh"
#include "sm100.cuh"

namespace gptq {
namespace {

using namespace sm100;

template <typename T>
__device__ __forceinline__ T from_f32(float v);
template <>
__device__ __forceinline__ __half from_f32<__half>(float v) { return __float2half_rn(v); }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

// round16(s * (q - z)) as a float, for 16-bit type T
template <typename T>
__device__ __forceinline__ float dq(float s, int q, int z) {
  return to_f32<T>(from_f32<T>(s * static_cast<float>(q - z)));
}

__device__ __forceinline__ int clamp_group(int g, int G) { return g < 0 ? 0 : (g >= G ? G - 1 : g); }

// ------------------------------------------------------------------ dequantization
// One CTA per 64 (k) x 64 (n) tile: dequantize into shared memory (reads coalesced along n),
// then write rows of W [N, K] (128 contiguous bytes per n, coalesced along k).
constexpr int DQ_T = 64;
template <int BITS, typename T>
__global__ void __launch_bounds__(256) dequant_kernel(const int32_t* __restrict__ qweight,
                                                      const int32_t* __restrict__ qzeros,
                                                      const __half* __restrict__ scales,
                                                      const int32_t* __restrict__ g_idx, int G, int64_t K,
                                                      int64_t N, T* __restrict__ W) {
  __shared__ __align__(16) T tile[DQ_T][DQ_T + 8];
  constexpr int FPW = 32 / BITS;
  constexpr uint32_t MASK = (1u << BITS) - 1u;
  const int64_t k0 = static_cast<int64_t>(blockIdx.x) * DQ_T, n0 = static_cast<int64_t>(blockIdx.y) * DQ_T;
  const int t = threadIdx.x;
  const int nl = t % DQ_T;
  const int kq = (t / DQ_T) * 16;  // 16 consecutive k per thread
  const int64_t n = n0 + nl;
  const int64_t zw = N * BITS / 32;
  if (n < N) {
    uint32_t word = 0;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int64_t k = k0 + kq + i;
      float v = 0.f;
      if (k < K) {
        if (i == 0 || (k % FPW) == 0) word = static_cast<uint32_t>(__ldg(qweight + (k / FPW) * N + n));
        const int q = static_cast<int>((word >> ((k % FPW) * BITS)) & MASK);
        const int g = clamp_group(__ldg(g_idx + k), G);
        const float s = __half2float(__ldg(scales + static_cast<int64_t>(g) * N + n));
        const uint32_t zword = static_cast<uint32_t>(__ldg(qzeros + static_cast<int64_t>(g) * zw + (n * BITS) / 32));
        const int z = static_cast<int>((zword >> ((n * BITS) % 32)) & MASK);
        v = dq<T>(s, q, z);
      }
      tile[nl][kq + i] = from_f32<T>(v);
    }
  }
  __syncthreads();
  // 64 rows x 8 chunks of 16 bytes
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int e = t + 256 * r;
    const int row = e / 8, ch = e % 8;
    const int64_t nn = n0 + row, kk = k0 + ch * 8;
    if (nn < N && kk < K)  // K % 8 == 0: a chunk is wholly inside or outside
      *reinterpret_cast<uint4*>(W + nn * K + kk) = *reinterpret_cast<const uint4*>(&tile[row][ch * 8]);
  }
}

// ------------------------------------------------------------------ tcgen05 GEMM, both operands K-major
constexpr int GBM = 128;  // rows of X per tile = UMMA M
constexpr int GBN = 256;  // output columns per tile = UMMA N
constexpr int GBK = 64;   // K per stage: one 128-byte swizzle row
constexpr int GSTAGES = 4;
constexpr int GA_BYTES = GBM * GBK * 2;
constexpr int GB_BYTES = GBN * GBK * 2;
constexpr int GSTAGE_BYTES = GA_BYTES + GB_BYTES;  // 48 KiB
constexpr int GTHREADS = 320;
constexpr int GSMEM = GSTAGES * GSTAGE_BYTES + 1024 + 256;
constexpr uint32_t GWAIT = 1u << 24;

__device__ int g_gemm_status = 0;

// Tile order: bands of GM row tiles; inside a band the row tile varies fastest, so a wave of
// CTAs covers GM row tiles x (wave / GM) column tiles and both operands' tiles of the wave
// stay in L2 (a band of X and a slice of the weight), instead of each wave streaming the
// whole weight for one row tile.
constexpr int GM_BAND = 16;
__device__ __forceinline__ void gemm_tile_at(int u, int mt, int nt, int& m_tile, int& n_tile) {
  const int band = u / (GM_BAND * nt);
  const int m_first = band * GM_BAND;
  const int bm = min(GM_BAND, mt - m_first);
  const int rem = u - band * GM_BAND * nt;
  n_tile = rem / bm;
  m_tile = m_first + rem % bm;
}

// K-major operand, 128-byte swizzle: rows of 64 16-bit elements (128 bytes), 8-row atoms of
// 1024 bytes (stride-dimension offset); the leading-dimension offset is unused because one
// MMA's K (16 elements, 32 bytes) lies inside a swizzle row.  K steps inside the row
// advance the start address by 32 bytes.
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t saddr) { return smem_desc_sw128(saddr, 16, 1024); }

template <uint32_t FMT, typename TOut>
__global__ void __launch_bounds__(GTHREADS, 1)
    gemm_tn_kernel(const __grid_constant__ CUtensorMap ta, const __grid_constant__ CUtensorMap tb,
                   TOut* __restrict__ Y, int M, int N, int K, int mt, int nt) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + GSTAGES * GSTAGE_BYTES);
  uint64_t* empty = full + GSTAGES;
  uint64_t* accf = empty + GSTAGES;
  uint64_t* acce = accf + 2;
  uint64_t* done = acce + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = static_cast<int>(gridDim.x);
  const int units = mt * nt;
  const int nk = (K + GBK - 1) / GBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < GSTAGES; ++s) {
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
      // ---------------- TMA producer
      tma_prefetch_desc(&ta);
      tma_prefetch_desc(&tb);
      int stage = 0, issued = 0;
      uint32_t ph = 0;
      for (int u = blockIdx.x; u < units && ok; u += G) {
        int mi, ni;
        gemm_tile_at(u, mt, nt, mi, ni);
        const int m0 = mi * GBM, n0 = ni * GBN;
        for (int ks = 0; ks < nk; ++ks) {
          if (!mbar_wait(&empty[stage], ph ^ 1u, GWAIT)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + stage * GSTAGE_BYTES;
          mbar_arrive_expect_tx(&full[stage], GSTAGE_BYTES);
          tma_load_2d(sa, &ta, &full[stage], ks * GBK, m0);
          tma_load_2d(sa + GA_BYTES, &tb, &full[stage], ks * GBK, n0);
          ++issued;
          if (++stage == GSTAGES) {
            stage = 0;
            ph ^= 1u;
          }
        }
      }
      // no copy of ours may still be landing in shared memory when the CTA leaves
      for (int k = 0; k < min(issued, GSTAGES); ++k) {
        int s = stage - 1 - k;
        uint32_t p = ph;
        while (s < 0) {
          s += GSTAGES;
          p ^= 1u;
        }
        mbar_wait(&full[s], p, GWAIT);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- UMMA issuer
      constexpr uint32_t idesc = instr_desc(FMT, false, false, GBM, GBN);
      int stage = 0, cg = 0;
      uint32_t ph = 0;
      for (int u = blockIdx.x; u < units && ok; u += G, ++cg) {
        const int b = cg & 1;
        if (!mbar_wait(&acce[b], ((cg >> 1) & 1) ^ 1u, GWAIT)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t dcol = tmem + static_cast<uint32_t>(b * GBN);
        for (int ks = 0; ks < nk; ++ks) {
          if (!mbar_wait(&full[stage], ph, GWAIT)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * GSTAGE_BYTES);
          const uint32_t sb = sa + GA_BYTES;
#pragma unroll
          for (int k = 0; k < GBK / 16; ++k)
            umma_f16(dcol, kmajor_desc(sa + k * 32), kmajor_desc(sb + k * 32), idesc, (ks > 0 || k > 0) ? 1u : 0u);
          umma_commit(&empty[stage]);
          if (++stage == GSTAGES) {
            stage = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;  // an incomplete accumulator is never handed to the epilogue
        umma_commit(&accf[b]);
      }
      umma_commit(done);
      mbar_wait(done, 0, GWAIT);
    }
  } else {
    // ---------------- epilogue (warps 2..9): TMEM -> registers -> 16-bit Y
    const int quad = warp & 3;         // TMEM lane quarter of this warp
    const int half = (warp - 2) >> 2;  // which 128 of the 256 columns
    int cg = 0;
    for (int u = blockIdx.x; u < units; u += G, ++cg) {
      const int b = cg & 1;
      if (!mbar_wait(&accf[b], (cg >> 1) & 1, GWAIT)) {
        ok = false;
        break;
      }
      tc_fence_after();
      int mi, ni;
      gemm_tile_at(u, mt, nt, mi, ni);
      const int m = mi * GBM + quad * 32 + lane;
      const int nb = ni * GBN + half * 128;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float v[32];
        tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(quad * 32) << 16) +
                               static_cast<uint32_t>(b * GBN + half * 128 + q * 32),
                           v);
        if (m < M) {
          TOut* yrow = Y + static_cast<int64_t>(m) * N;
#pragma unroll
          for (int c8 = 0; c8 < 4; ++c8) {
            const int n = nb + q * 32 + c8 * 8;
            if (n < N) {  // N % 8 == 0: an 8-column chunk is wholly inside or outside
              alignas(16) TOut o[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) o[e] = from_f32<TOut>(v[c8 * 8 + e]);
              *reinterpret_cast<uint4*>(yrow + n) = *reinterpret_cast<const uint4*>(o);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acce[b]);
    }
  }
  if (!ok) atomicExch(&g_gemm_status, kStatusTimeout);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ decode GEMV (M <= 4)
constexpr int GV_THREADS = 256;  // 8 warps; a lane owns 4 consecutive outputs
constexpr int GV_N = 128;        // outputs per CTA
constexpr int GV_MAXM = 4;
constexpr int GV_ROWS = 4;       // word rows of one warp in flight

// Packed fp32 pairs (the f32x2 arithmetic of sm_100).
__device__ __forceinline__ unsigned long long f2_bits(float2 v) { return *reinterpret_cast<unsigned long long*>(&v); }
__device__ __forceinline__ float2 bits_f2(unsigned long long b) { return *reinterpret_cast<float2*>(&b); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(f2_bits(a)), "l"(f2_bits(b)), "l"(f2_bits(c)));
  return bits_f2(d);
}
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
  unsigned long long d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(f2_bits(a)), "l"(f2_bits(b)));
  return bits_f2(d);
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  unsigned long long d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(f2_bits(a)), "l"(f2_bits(b)));
  return bits_f2(d);
}

// Group parameters of one output in the form the paired dequantization wants, and the
// pair itself: codes i and i + FPW/2 of a word (the same bit offset in its two 16-bit
// halves), both returned as round16(s * (q - z)) in a float2.
//  * float16: 0x6400 | q is the half 1024 + q (exact for q < 1024); subtracting 1024 + z
//    leaves q - z exactly, and one half multiply by s rounds the exact product once, to
//    nearest even: round16(s * (q - z)), two codes per instruction.
//  * bfloat16: the same with bf16 pairs, the scale split in two bf16 parts so that one
//    fused multiply-add rounds the exact product once (8-bit codes: in fp32, 0x4B000000 | q
//    being 2^23 + q, then one rounding to bfloat16).
template <typename T>
struct PairDeq;
template <>
struct PairDeq<__half> {
  __half2 s2, zb2;
  __device__ __forceinline__ void set(float s, int z) {
    s2 = __float2half2_rn(s);  // s is a float16 value: exact
    zb2 = __float2half2_rn(1024.f + static_cast<float>(z));
  }
  template <int BITS>
  __device__ __forceinline__ float2 pair(uint32_t w, int i) const {
    constexpr uint32_t m = (1u << BITS) - 1u;
    const uint32_t h = ((w >> (i * BITS)) & ((m << 16) | m)) | 0x64006400u;
    const __half2 v = __hmul2(__hsub2(*reinterpret_cast<const __half2*>(&h), zb2), s2);
    return __half22float2(v);
  }
};
template <>
struct PairDeq<__nv_bfloat16> {
  // codes of up to 4 bits: s = s_hi + s_lo with s_hi = bf16(s) and s_lo (at most 3 bits) both
  // exact in bf16; 0x4300 | q is the bf16 128 + q, so d = q - z is exact, s_lo d is exact (at
  // most 7 bits) and one bf16 FMA s_hi d + s_lo d rounds the exact product once
  __nv_bfloat162 shi2, slo2, zb2;
  // 8-bit codes (q - z needs 9 bits): the fp32 route, exact up to one rounding to bf16
  float2 s2, zf2;
  __device__ __forceinline__ void set(float s, int z) {
    const __nv_bfloat16 hi = __float2bfloat16_rn(s);
    shi2 = __bfloat162bfloat162(hi);
    slo2 = __bfloat162bfloat162(__float2bfloat16_rn(s - __bfloat162float(hi)));
    zb2 = __bfloat162bfloat162(__float2bfloat16_rn(128.f + static_cast<float>(z)));
    s2 = make_float2(s, s);
    zf2 = make_float2(8388608.f + static_cast<float>(z), 8388608.f + static_cast<float>(z));
  }
  template <int BITS>
  __device__ __forceinline__ float2 pair(uint32_t w, int i) const {
    constexpr uint32_t m = (1u << BITS) - 1u;
    if constexpr (BITS <= 4) {
      const uint32_t h = ((w >> (i * BITS)) & ((m << 16) | m)) | 0x43004300u;
      const __nv_bfloat162 d = __hsub2(*reinterpret_cast<const __nv_bfloat162*>(&h), zb2);
      return __bfloat1622float2(__hfma2(shi2, d, __hmul2(slo2, d)));
    } else {
      const uint32_t lo = (w >> (i * BITS)) & m, hi = (w >> (i * BITS + 16)) & m;
      const float2 q = make_float2(__uint_as_float(0x4B000000u | lo), __uint_as_float(0x4B000000u | hi));
      return __bfloat1622float2(__float22bfloat162_rn(mul2(sub2(q, zf2), s2)));
    }
  }
};

// One CTA: 128 outputs x one K chunk.  The chunk's activations are staged in shared memory
// as pairs (x[k], x[k + FPW/2]) matching the paired codes, and every word row is marked
// with its group when all its FPW codes share one (always for checkpoints whose g_idx runs
// in order), else -1.  Rows of one group take the paired path with the group parameters
// loaded once per group; mixed rows (act-order checkpoints) take a per-code path with a
// group lookup for every code.  Each warp keeps GV_ROWS word rows in flight (16-byte loads,
// a warp reads 512 contiguous bytes of a row); fp32 products are accumulated in pairs.
template <int BITS, typename T, int MM>
__global__ void __launch_bounds__(GV_THREADS, 2) gemv_kernel(const T* __restrict__ X, int M, int64_t K,
                                                          const int32_t* __restrict__ qweight,
                                                          const int32_t* __restrict__ qzeros,
                                                          const __half* __restrict__ scales,
                                                          const int32_t* __restrict__ g_idx,
                                                          const int32_t* __restrict__ x_perm, int G, int64_t N,
                                                          int kchunk, float* __restrict__ partial) {
  constexpr int FPW = 32 / BITS;
  constexpr int HP = FPW / 2;  // code pairs per word
  constexpr uint32_t MASK = (1u << BITS) - 1u;
  extern __shared__ __align__(16) float gsm[];
  float2* xs = reinterpret_cast<float2*>(gsm);            // [MM][kchunk / 2] pairs
  int* gs = reinterpret_cast<int*>(gsm + MM * kchunk);     // [kchunk] group of each k
  int* rg = gs + kchunk;                                   // [kchunk / FPW] group of each row
  float* red = reinterpret_cast<float*>(rg + kchunk / 4);  // [8][MM][GV_N] (FPW >= 4)
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t klo = static_cast<int64_t>(blockIdx.y) * kchunk;
  const int kn = static_cast<int>(min(static_cast<int64_t>(kchunk), K - klo));
  const int rows = kn / FPW;  // kchunk and K are multiples of FPW
  for (int e = tid; e < kn; e += GV_THREADS) {
    gs[e] = clamp_group(__ldg(g_idx + klo + e), G);
    // k = r*FPW + f sits in pair slot r*HP + (f mod HP), component f / HP
    const int r = e / FPW, f = e % FPW;
    float* slot = reinterpret_cast<float*>(xs + r * HP + (f % HP)) + (f / HP);
#pragma unroll
    // the input behind row k of the codes (clamped: a malformed permutation reads inside X)
    const int64_t kx = x_perm ? min(max(static_cast<int64_t>(__ldg(x_perm + klo + e)), int64_t(0)), K - 1) : klo + e;
#pragma unroll
    for (int m = 0; m < MM; ++m) slot[m * kchunk] = to_f32<T>(X[m * K + kx]);
  }
  __syncthreads();
  for (int r = tid; r < rows; r += GV_THREADS) {
    const int g0 = gs[r * FPW];
    bool same = true;
#pragma unroll
    for (int f = 1; f < FPW; ++f) same = same && gs[r * FPW + f] == g0;
    rg[r] = same ? g0 : -1;
  }
  __syncthreads();
  const int64_t n = static_cast<int64_t>(blockIdx.x) * GV_N + lane * 4;
  float2 acc[MM][4];
#pragma unroll
  for (int m = 0; m < MM; ++m)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[m][j] = make_float2(0.f, 0.f);
  if (n < N) {
    const int64_t zw = N * BITS / 32;
    const int zshift = static_cast<int>((n * BITS) % 32);
    int gcur = -1, gpair = -1;  // group of sc/zc, group of pd
    PairDeq<T> pd[4];
    float sc[4];
    int zc[4];
    auto load_group = [&](int g) {
      gcur = g;
      const uint2 s4 = __ldg(reinterpret_cast<const uint2*>(scales + static_cast<int64_t>(g) * N + n));
      const __half2 s01 = *reinterpret_cast<const __half2*>(&s4.x);
      const __half2 s23 = *reinterpret_cast<const __half2*>(&s4.y);
      sc[0] = __low2float(s01);
      sc[1] = __high2float(s01);
      sc[2] = __low2float(s23);
      sc[3] = __high2float(s23);
      const uint32_t zword = static_cast<uint32_t>(__ldg(qzeros + static_cast<int64_t>(g) * zw + (n * BITS) / 32));
#pragma unroll
      for (int j = 0; j < 4; ++j) zc[j] = static_cast<int>((zword >> (zshift + j * BITS)) & MASK);
    };
    auto row_math = [&](int r, const int4 w4) {
      const uint32_t wv[4] = {static_cast<uint32_t>(w4.x), static_cast<uint32_t>(w4.y), static_cast<uint32_t>(w4.z),
                              static_cast<uint32_t>(w4.w)};
      const int g = rg[r];
      if (g >= 0) {
        if (g != gpair) {
          if (g != gcur) load_group(g);
#pragma unroll
          for (int j = 0; j < 4; ++j) pd[j].set(sc[j], zc[j]);
          gpair = g;
        }
#pragma unroll
        for (int i = 0; i < HP; ++i) {
          float2 xp[MM];
#pragma unroll
          for (int m = 0; m < MM; ++m) xp[m] = xs[m * (kchunk / 2) + r * HP + i];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float2 w = pd[j].template pair<BITS>(wv[j], i);
#pragma unroll
            for (int m = 0; m < MM; ++m) acc[m][j] = fma2(xp[m], w, acc[m][j]);
          }
        }
      } else {
        // mixed groups within the row: one code at a time
#pragma unroll
        for (int f = 0; f < FPW; ++f) {
          const int gk = gs[r * FPW + f];
          if (gk != gcur) load_group(gk);
          const int slot = r * HP + (f % HP);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float w = dq<T>(sc[j], static_cast<int>((wv[j] >> (f * BITS)) & MASK), zc[j]);
#pragma unroll
            for (int m = 0; m < MM; ++m) {
              const float x = reinterpret_cast<const float*>(xs + m * (kchunk / 2) + slot)[f / HP];
              if (f / HP == 0)
                acc[m][j].x = fmaf(x, w, acc[m][j].x);
              else
                acc[m][j].y = fmaf(x, w, acc[m][j].y);
            }
          }
        }
      }
    };
    const int64_t wbase = klo / FPW;
    constexpr int RF = BITS == 2 ? 2 : GV_ROWS;  // 2-bit rows unpack twice the codes
    int r = warp;
    for (; r + 8 * (RF - 1) < rows; r += 8 * RF) {
      int4 w[RF];
#pragma unroll
      for (int t = 0; t < RF; ++t)
        w[t] = __ldg(reinterpret_cast<const int4*>(qweight + (wbase + r + 8 * t) * N + n));
#pragma unroll
      for (int t = 0; t < RF; ++t) row_math(r + 8 * t, w[t]);
    }
    for (; r < rows; r += 8) row_math(r, __ldg(reinterpret_cast<const int4*>(qweight + (wbase + r) * N + n)));
  }
  // the 8 warps' partial sums of this CTA's outputs, added in a fixed order
#pragma unroll
  for (int m = 0; m < MM; ++m)
#pragma unroll
    for (int j = 0; j < 4; ++j) red[(warp * MM + m) * GV_N + lane * 4 + j] = acc[m][j].x + acc[m][j].y;
  __syncthreads();
  for (int e = tid; e < MM * GV_N; e += GV_THREADS) {
    const int m = e / GV_N, c = e % GV_N;
    const int64_t nn = static_cast<int64_t>(blockIdx.x) * GV_N + c;
    if (m < M && nn < N) {
      float t = 0.f;
      for (int w = 0; w < 8; ++w) t += red[(w * MM + m) * GV_N + c];
      partial[(static_cast<int64_t>(blockIdx.y) * M + m) * N + nn] = t;
    }
  }
}

// ------------------------------------------------------------------ act-order reordering
// A checkpoint quantized with act order stores its codes in the original input order, with
// g_idx naming each input's group; the inputs of a 32-bit word then belong to different
// groups.  Reordering the inputs by group (and gathering X by the same permutation) gives a
// checkpoint whose g_idx runs in order, which the decode kernel dequantizes two codes at a
// time; the product is the same sum over the inputs in another order.
//
// perm[k'] = the input with the k'-th smallest (g_idx, index): one CTA of 1024 threads, the
// group sizes in shared memory, their exclusive scan, then the inputs in chunks of 1024 in
// increasing index, each placed at its group's running offset plus its rank among the chunk's
// inputs of the same group (stable, deterministic).
constexpr int RO_THREADS = 1024;
__global__ void __launch_bounds__(RO_THREADS) sort_by_group_kernel(const int32_t* __restrict__ g_idx, int K, int G,
                                                                   int32_t* __restrict__ perm,
                                                                   int32_t* __restrict__ g_sorted) {
  extern __shared__ int ro_sm[];
  int* off = ro_sm;             // [G] group sizes, then running offsets
  int* gch = ro_sm + G;         // [RO_THREADS] groups of the current chunk
  int* part = gch + RO_THREADS; // [RO_THREADS] per-thread partial sums of the scan
  const int tid = threadIdx.x;
  for (int g = tid; g < G; g += RO_THREADS) off[g] = 0;
  __syncthreads();
  for (int k = tid; k < K; k += RO_THREADS) atomicAdd(&off[clamp_group(g_idx[k], G)], 1);
  __syncthreads();
  // exclusive scan: each thread a contiguous range, then the range totals by thread 0
  const int per = (G + RO_THREADS - 1) / RO_THREADS;
  const int lo = min(G, tid * per), hi = min(G, lo + per);
  int sum = 0;
  for (int g = lo; g < hi; ++g) sum += off[g];
  part[tid] = sum;
  __syncthreads();
  if (tid == 0) {
    int run = 0;
    for (int t = 0; t < RO_THREADS; ++t) {
      const int v = part[t];
      part[t] = run;
      run += v;
    }
  }
  __syncthreads();
  int run = part[tid];
  for (int g = lo; g < hi; ++g) {
    const int v = off[g];
    off[g] = run;
    run += v;
  }
  __syncthreads();
  for (int c0 = 0; c0 < K; c0 += RO_THREADS) {
    const int k = c0 + tid;
    const int g = k < K ? clamp_group(g_idx[k], G) : -1;
    gch[tid] = g;
    __syncthreads();
    int rank = 0;
    bool last = true;
    if (g >= 0) {
      for (int j = 0; j < RO_THREADS; ++j) {
        const int gj = gch[j];
        rank += (j < tid && gj == g) ? 1 : 0;
        last = last && !(j > tid && gj == g);
      }
      const int pos = off[g] + rank;
      perm[pos] = k;
      g_sorted[pos] = g;
    }
    __syncthreads();  // every rank and offset read before the offsets move on
    if (g >= 0 && last) off[g] += rank + 1;  // the group's last input of the chunk
    __syncthreads();
  }
}

// Word row r' of the reordered codes holds inputs perm[r' FPW .. r' FPW + FPW - 1].
template <int BITS>
__global__ void reorder_codes_kernel(const int32_t* __restrict__ qweight, const int32_t* __restrict__ perm,
                                     int64_t rows, int64_t N, int32_t* __restrict__ out) {
  constexpr int FPW = 32 / BITS;
  constexpr uint32_t MASK = (1u << BITS) - 1u;
  const int64_t n = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t r = blockIdx.y;
  if (n >= N || r >= rows) return;
  uint32_t w = 0;
#pragma unroll
  for (int f = 0; f < FPW; ++f) {
    const int k = perm[r * FPW + f];
    const uint32_t src = static_cast<uint32_t>(__ldg(qweight + static_cast<int64_t>(k / FPW) * N + n));
    w |= ((src >> ((k % FPW) * BITS)) & MASK) << (f * BITS);
  }
  out[r * N + n] = static_cast<int32_t>(w);
}

// X'[m, k'] = X[m, perm[k']] for the tensor-core path.
template <typename T>
__global__ void gather_cols_kernel(const T* __restrict__ X, const int32_t* __restrict__ perm, int64_t M, int64_t K,
                                   T* __restrict__ Xp) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= M * K) return;
  const int64_t m = i / K, k = i % K;
  const int64_t kx = min(max(static_cast<int64_t>(perm[k]), int64_t(0)), K - 1);
  Xp[i] = X[m * K + kx];
}

// Y[m, n] = sum over K splits of partial[s, m, n], in split order.
template <typename T>
__global__ void split_sum_kernel(const float* __restrict__ partial, int S, int M, int64_t N, T* __restrict__ Y) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= static_cast<int64_t>(M) * N) return;
  float t = 0.f;
  for (int s = 0; s < S; ++s) t += partial[static_cast<int64_t>(s) * M * N + i];
  Y[i] = from_f32<T>(t);
}

// ------------------------------------------------------------------ host side
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

// rows x K (K contiguous) 16-bit matrix, boxes of 64 (K) x box_rows, 128-byte swizzle
int kmajor_map(CUtensorMap* tm, const void* base, int bf16, int64_t rows, int64_t K, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return GPTQ_ERR_CUDA;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
  cuuint32_t box[2] = {GBK, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(tm, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
                         const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? GPTQ_OK : GPTQ_ERR_CUDA;
}

template <uint32_t FMT, typename T>
int launch_gemm(const T* X, const T* Wd, T* Y, int64_t M, int64_t N, int64_t K, cudaStream_t s) {
  GPTQ_TRY(ensure_smem_limit(reinterpret_cast<const void*>(gemm_tn_kernel<FMT, T>), GSMEM));
  CUtensorMap ta, tb;
  GPTQ_TRY(kmajor_map(&ta, X, FMT == 1, M, K, GBM));
  GPTQ_TRY(kmajor_map(&tb, Wd, FMT == 1, N, K, GBN));
  const int64_t mt = (M + GBM - 1) / GBM, nt = (N + GBN - 1) / GBN;
  if (mt * nt >= (int64_t(1) << 31)) return GPTQ_ERR_UNSUPPORTED;
  const int grid = static_cast<int>(std::min<int64_t>(num_sms(), mt * nt));
  gemm_tn_kernel<FMT, T><<<grid, GTHREADS, GSMEM, s>>>(ta, tb, Y, static_cast<int>(M), static_cast<int>(N),
                                                       static_cast<int>(K), static_cast<int>(mt), static_cast<int>(nt));
  return after_launch();
}

template <int BITS, typename T>
int launch_dequant(const int32_t* qweight, const int32_t* qzeros, const __half* scales, const int32_t* g_idx, int G,
                   int64_t K, int64_t N, T* W, cudaStream_t s) {
  const dim3 grid(static_cast<unsigned>((K + DQ_T - 1) / DQ_T), static_cast<unsigned>((N + DQ_T - 1) / DQ_T));
  dequant_kernel<BITS, T><<<grid, 256, 0, s>>>(qweight, qzeros, scales, g_idx, G, K, N, W);
  return after_launch();
}

template <typename T>
int dequant_any(int bits, const int32_t* qw, const int32_t* qz, const __half* sc, const int32_t* gi, int G, int64_t K,
                int64_t N, T* W, cudaStream_t s) {
  if (bits == 2) return launch_dequant<2, T>(qw, qz, sc, gi, G, K, N, W, s);
  if (bits == 4) return launch_dequant<4, T>(qw, qz, sc, gi, G, K, N, W, s);
  return launch_dequant<8, T>(qw, qz, sc, gi, G, K, N, W, s);
}

template <int BITS, typename T, int MM>
int launch_gemv(const T* X, int M, int64_t K, const int32_t* qw, const int32_t* qz, const __half* sc,
                const int32_t* gi, const int32_t* xp, int G, int64_t N, T* Y, cudaStream_t s) {
  // K split so that about four CTAs per SM stream the weights; every split a multiple of
  // 64 columns (whole words for every bit width).
  const int64_t nblk = (N + GV_N - 1) / GV_N;
  int64_t S = std::max<int64_t>(1, (4 * num_sms() + nblk - 1) / nblk);
  int64_t kchunk = std::max<int64_t>(64, (((K + S - 1) / S) + 63) / 64 * 64);
  kchunk = std::min<int64_t>(kchunk, 4096);
  S = (K + kchunk - 1) / kchunk;
  if (S > 65535) return GPTQ_ERR_UNSUPPORTED;
  const size_t smem = (MM * kchunk + kchunk + kchunk / 4) * 4 + 8 * MM * GV_N * 4;
  GPTQ_TRY(ensure_smem_limit(reinterpret_cast<const void*>(gemv_kernel<BITS, T, MM>), static_cast<int>(smem)));
  float* partial = nullptr;
  GPTQ_TRY(pool_alloc(reinterpret_cast<void**>(&partial), static_cast<size_t>(S) * M * N * 4, s));
  gemv_kernel<BITS, T, MM><<<dim3(static_cast<unsigned>(nblk), static_cast<unsigned>(S)), GV_THREADS, smem, s>>>(
      X, M, K, qw, qz, sc, gi, xp, G, N, static_cast<int>(kchunk), partial);
  int st = after_launch();
  if (st == GPTQ_OK) {
    const int64_t cnt = static_cast<int64_t>(M) * N;
    split_sum_kernel<T><<<static_cast<unsigned>((cnt + 255) / 256), 256, 0, s>>>(partial, static_cast<int>(S), M, N, Y);
    st = after_launch();
  }
  pool_free(partial, s);
  return st;
}

template <int BITS, typename T>
int gemv_rows(const T* X, int M, int64_t K, const int32_t* qw, const int32_t* qz, const __half* sc,
              const int32_t* gi, const int32_t* xp, int G, int64_t N, T* Y, cudaStream_t s) {
  switch (M) {
    case 1: return launch_gemv<BITS, T, 1>(X, M, K, qw, qz, sc, gi, xp, G, N, Y, s);
    case 2: return launch_gemv<BITS, T, 2>(X, M, K, qw, qz, sc, gi, xp, G, N, Y, s);
    case 3: return launch_gemv<BITS, T, 3>(X, M, K, qw, qz, sc, gi, xp, G, N, Y, s);
    default: return launch_gemv<BITS, T, 4>(X, M, K, qw, qz, sc, gi, xp, G, N, Y, s);
  }
}

template <typename T>
int gemv_any(int bits, const T* X, int M, int64_t K, const int32_t* qw, const int32_t* qz, const __half* sc,
             const int32_t* gi, const int32_t* xp, int G, int64_t N, T* Y, cudaStream_t s) {
  if (bits == 2) return gemv_rows<2, T>(X, M, K, qw, qz, sc, gi, xp, G, N, Y, s);
  if (bits == 4) return gemv_rows<4, T>(X, M, K, qw, qz, sc, gi, xp, G, N, Y, s);
  return gemv_rows<8, T>(X, M, K, qw, qz, sc, gi, xp, G, N, Y, s);
}

int check_qlinear(const int32_t* qweight, const int32_t* qzeros, const uint16_t* scales, const int32_t* g_idx,
                  int64_t groups, int64_t n_in, int64_t n_out, int bits) {
  if (!qweight || !qzeros || !scales || !g_idx) return GPTQ_ERR_INVALID_ARG;
  if (n_in <= 0 || n_out <= 0 || groups <= 0) return GPTQ_ERR_INVALID_ARG;
  if (bits != 2 && bits != 3 && bits != 4 && bits != 8) return GPTQ_ERR_INVALID_ARG;
  if (bits == 3) return GPTQ_ERR_UNSUPPORTED;  // fields straddle words; not handled here
  // whole 32-bit words of zero points per group (n_out * bits % 32), 16-byte output rows
  if (n_in % 64 != 0 || n_out % 8 != 0 || (n_out * bits) % 32 != 0 || groups > n_in || n_in > (int64_t(1) << 30) ||
      n_out > (int64_t(1) << 30))
    return GPTQ_ERR_UNSUPPORTED;
  if (!aligned16(qweight) || !aligned16(qzeros) || !aligned16(scales) || !aligned16(g_idx)) return GPTQ_ERR_UNSUPPORTED;
  return GPTQ_OK;
}

}  // namespace

int gemm_bf16_tn(const void* X, const void* Wd, void* Y, int64_t M, int64_t N, int64_t K, int x_dtype,
                 cudaStream_t s) {
  if (x_dtype == GPTQ_BF16)
    return launch_gemm<1, __nv_bfloat16>(static_cast<const __nv_bfloat16*>(X), static_cast<const __nv_bfloat16*>(Wd),
                                         static_cast<__nv_bfloat16*>(Y), M, N, K, s);
  return launch_gemm<0, __half>(static_cast<const __half*>(X), static_cast<const __half*>(Wd), static_cast<__half*>(Y),
                                M, N, K, s);
}

int gemm_device_status(int clear) {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_gemm_status, sizeof(int)) != cudaSuccess) return GPTQ_ERR_CUDA;
  if (clear) {
    int z = 0;
    if (cudaMemcpyToSymbol(g_gemm_status, &z, sizeof(int)) != cudaSuccess) return GPTQ_ERR_CUDA;
  }
  return v;
}

}  // namespace gptq

using namespace gptq;

extern "C" int gptq_dequantize_weight(const int32_t* qweight, const int32_t* qzeros, const uint16_t* scales_f16,
                                      const int32_t* g_idx, int64_t groups, int64_t n_in, int64_t n_out, int bits,
                                      int out_dtype, void* W, void* stream) {
  GPTQ_TRY(check_qlinear(qweight, qzeros, scales_f16, g_idx, groups, n_in, n_out, bits));
  if (!W) return GPTQ_ERR_INVALID_ARG;
  if (out_dtype != GPTQ_F16 && out_dtype != GPTQ_BF16) return GPTQ_ERR_INVALID_ARG;
  if (!aligned16(W)) return GPTQ_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const __half* sc = reinterpret_cast<const __half*>(scales_f16);
  const int G = static_cast<int>(groups);
  if (out_dtype == GPTQ_BF16)
    return dequant_any<__nv_bfloat16>(bits, qweight, qzeros, sc, g_idx, G, n_in, n_out, static_cast<__nv_bfloat16*>(W), s);
  return dequant_any<__half>(bits, qweight, qzeros, sc, g_idx, G, n_in, n_out, static_cast<__half*>(W), s);
}

extern "C" int gptq_quantized_linear(const void* X, int x_dtype, int64_t M, int64_t n_in, const int32_t* qweight,
                                     const int32_t* qzeros, const uint16_t* scales_f16, const int32_t* g_idx,
                                     const int32_t* x_perm, int64_t groups, int64_t n_out, int bits, void* Y,
                                     void* stream) {
  GPTQ_TRY(check_qlinear(qweight, qzeros, scales_f16, g_idx, groups, n_in, n_out, bits));
  if (M < 0 || ((!X || !Y) && M > 0)) return GPTQ_ERR_INVALID_ARG;  // no rows: X and Y may be NULL
  if (x_dtype != GPTQ_F16 && x_dtype != GPTQ_BF16) return GPTQ_ERR_INVALID_ARG;
  if (M == 0) return GPTQ_OK;
  if (M >= (int64_t(1) << 31)) return GPTQ_ERR_UNSUPPORTED;
  if (!aligned16(X) || !aligned16(Y) || (x_perm && !aligned16(x_perm))) return GPTQ_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const __half* sc = reinterpret_cast<const __half*>(scales_f16);
  const int G = static_cast<int>(groups);
  if (M <= GV_MAXM) {
    if (x_dtype == GPTQ_BF16)
      return gemv_any<__nv_bfloat16>(bits, static_cast<const __nv_bfloat16*>(X), static_cast<int>(M), n_in, qweight,
                                     qzeros, sc, g_idx, x_perm, G, n_out, static_cast<__nv_bfloat16*>(Y), s);
    return gemv_any<__half>(bits, static_cast<const __half*>(X), static_cast<int>(M), n_in, qweight, qzeros, sc, g_idx,
                            x_perm, G, n_out, static_cast<__half*>(Y), s);
  }
  const size_t xbytes = x_perm ? static_cast<size_t>(M) * n_in * 2 : 0;
  void* Wd = nullptr;
  GPTQ_TRY(pool_alloc(&Wd, static_cast<size_t>(n_in) * n_out * 2 + xbytes, s));
  const void* Xg = X;
  int st = GPTQ_OK;
  if (x_perm) {  // X with its columns in the order of the codes
    void* Xp = static_cast<char*>(Wd) + static_cast<size_t>(n_in) * n_out * 2;
    const int64_t cnt = M * n_in;
    const unsigned gx = static_cast<unsigned>((cnt + 255) / 256);
    if (x_dtype == GPTQ_BF16)
      gather_cols_kernel<__nv_bfloat16><<<gx, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(X), x_perm, M, n_in,
                                                           static_cast<__nv_bfloat16*>(Xp));
    else
      gather_cols_kernel<__half><<<gx, 256, 0, s>>>(static_cast<const __half*>(X), x_perm, M, n_in,
                                                    static_cast<__half*>(Xp));
    st = after_launch();
    Xg = Xp;
  }
  if (st == GPTQ_OK)
    st = x_dtype == GPTQ_BF16
             ? dequant_any<__nv_bfloat16>(bits, qweight, qzeros, sc, g_idx, G, n_in, n_out,
                                          static_cast<__nv_bfloat16*>(Wd), s)
             : dequant_any<__half>(bits, qweight, qzeros, sc, g_idx, G, n_in, n_out, static_cast<__half*>(Wd), s);
  if (st == GPTQ_OK) st = gemm_bf16_tn(Xg, Wd, Y, M, n_out, n_in, x_dtype, s);
  pool_free(Wd, s);
  return st;
}

extern "C" int gptq_reorder_act_order(const int32_t* qweight, const int32_t* g_idx, int64_t groups, int64_t n_in,
                                      int64_t n_out, int bits, int32_t* qweight_out, int32_t* g_idx_out,
                                      int32_t* x_perm, void* stream) {
  if (!qweight || !g_idx || !qweight_out || !g_idx_out || !x_perm) return GPTQ_ERR_INVALID_ARG;
  if (n_in <= 0 || n_out <= 0 || groups <= 0) return GPTQ_ERR_INVALID_ARG;
  if (bits != 2 && bits != 3 && bits != 4 && bits != 8) return GPTQ_ERR_INVALID_ARG;
  if (bits == 3) return GPTQ_ERR_UNSUPPORTED;
  // the group counters live in shared memory: at most 32768 groups
  if (n_in % 64 != 0 || groups > n_in || groups > 32768 || n_in > 65536 || n_out > (int64_t(1) << 30))
    return GPTQ_ERR_UNSUPPORTED;
  if (qweight == qweight_out || g_idx == g_idx_out) return GPTQ_ERR_INVALID_ARG;  // not in place
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int G = static_cast<int>(groups), K = static_cast<int>(n_in);
  const int smem = (G + 2 * RO_THREADS) * static_cast<int>(sizeof(int));
  GPTQ_TRY(ensure_smem_limit(reinterpret_cast<const void*>(sort_by_group_kernel), smem));
  sort_by_group_kernel<<<1, RO_THREADS, smem, s>>>(g_idx, K, G, x_perm, g_idx_out);
  GPTQ_TRY(after_launch());
  const int64_t rows = n_in * bits / 32;
  const dim3 grid(static_cast<unsigned>((n_out + 255) / 256), static_cast<unsigned>(rows));
  if (bits == 2)
    reorder_codes_kernel<2><<<grid, 256, 0, s>>>(qweight, x_perm, rows, n_out, qweight_out);
  else if (bits == 4)
    reorder_codes_kernel<4><<<grid, 256, 0, s>>>(qweight, x_perm, rows, n_out, qweight_out);
  else
    reorder_codes_kernel<8><<<grid, 256, 0, s>>>(qweight, x_perm, rows, n_out, qweight_out);
  return after_launch();
}
